// prefix.cuh -- sequential temperature scaling, survival and the greedy
// hardware-aware prefix cut, in one CTA.
//
// The whole batch has at most kMaxCand = 8192 candidates (B*K), ordered by
// survival descending, ties by candidate index k*B + b ascending (position
// then request).  Survival never rises along a request's positions (each
// step multiplies by c in (0, 1]), so each request's K candidates are
// already a sorted run.  Blocks of 256 or 512 candidates are sorted by one
// warp each (a bitonic network in registers and shuffles), then merged as a
// tree in shared memory (each thread finds its output chunk's split by a
// merge-path binary search, then merges it sequentially).  The buffers carry the survival keys with the candidate ids: an earlier form
// that merged ids and looked every key up by id spent 65 of its 86 us at
// the stress shape in the merge.  The
// expected-emitted-token prefix sums are a block scan in fp64, and the early
// stop is the first index where E/t(N) does not increase.
//
// Asynchronous budget (yage.ai, engineering paragraph: how many tokens a
// step verifies is decided from the confidences of two steps back, which
// tokens fill that budget from the current ones): with a budget of N verify
// tokens the first N - B candidates of the current order are committed;
// the greedy N of the current confidences is returned either way, to be the
// budget two steps later.  The budget is read before the new one is
// written, so the two may share one device word.  The cost table can be
// read piecewise-linearly or as a staircase (the same page: the measured
// throughput curve jumps in steps).
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kPrefixThreads = 1024;
constexpr int kPrefixThreadsSmall = 128;   // for at most kPrefixSmallCand candidates
constexpr int kPrefixSmallCand = 1024;
constexpr int kMaxCand = 8192;

// Piecewise-linear cost (ms) of a verify batch of n tokens, extended
// linearly past both ends of the table.
__device__ __forceinline__ double cost_at(const float* __restrict__ xs, const float* __restrict__ ys,
                                          int n, double tokens) {
  int i = 0;
  while (i < n - 2 && tokens > (double)xs[i + 1]) ++i;
  const double x0 = xs[i], x1 = xs[i + 1], y0 = ys[i], y1 = ys[i + 1];
  return y0 + (y1 - y0) * (tokens - x0) / (x1 - x0);
}

// Staircase reading: the entry of the smallest profiled size that holds the
// batch; past the table, the last segment's slope.
__device__ __forceinline__ double cost_stair_at(const float* __restrict__ xs,
                                                const float* __restrict__ ys, int n,
                                                double tokens) {
  if (tokens > (double)xs[n - 1])
    return (double)ys[n - 1] + ((double)ys[n - 1] - (double)ys[n - 2]) *
                                   (tokens - (double)xs[n - 1]) /
                                   ((double)xs[n - 1] - (double)xs[n - 2]);
  int i = 0;
  while ((double)xs[i] < tokens) ++i;
  return ys[i];
}

__device__ __forceinline__ double cost_of(const float* __restrict__ xs, const float* __restrict__ ys,
                                          int n, int staircase, double tokens) {
  return staircase ? cost_stair_at(xs, ys, n, tokens) : cost_at(xs, ys, n, tokens);
}

// cost_of for a non-decreasing sequence of token counts: the table position
// only moves forward, so each lookup is amortised O(1).  Same arithmetic and
// results as cost_of.
struct CostWalker {
  const float* xs;
  const float* ys;
  int n, staircase, i;
  __device__ double at(double tokens) {
    if (staircase) {
      if (tokens > (double)xs[n - 1]) return cost_stair_at(xs, ys, n, tokens);
      while ((double)xs[i] < tokens) ++i;
      return ys[i];
    }
    while (i < n - 2 && tokens > (double)xs[i + 1]) ++i;
    const double x0 = xs[i], x1 = xs[i + 1], y0 = ys[i], y1 = ys[i + 1];
    return y0 + (y1 - y0) * (tokens - x0) / (x1 - x0);
  }
};

// key order: larger survival first; equal survival: smaller index first
__device__ __forceinline__ bool cand_before(double sa, int ia, double sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

// Sorts the elements [e0, e0 + 32 kE) of (key, idx) in place by cand_before
// with a bitonic network run by one warp: lane l holds elements e0 + kE l ..
// e0 + kE l + kE - 1 in registers; exchanges at distances below kE stay
// inside a lane, longer ones cross lanes by shuffles.  Elements at or past
// n are padding that sorts last and is not written back.  cand_before is a
// strict total order on distinct ids, so the result is the unique sorted
// order.
template <int kE>
__device__ __forceinline__ void warp_sort(double* key, int* idx, int e0, int n) {
  constexpr int kN = 32 * kE;
  const int lane = threadIdx.x & 31;
  double kv[kE];
  int iv[kE];
#pragma unroll
  for (int i = 0; i < kE; ++i) {
    const int e = e0 + kE * lane + i;
    kv[i] = e < n ? key[e] : -1.0;  // survivals are >= 0
    iv[i] = e < n ? idx[e] : 0x7fffffff;
  }
#pragma unroll
  for (int sz = 2; sz <= kN; sz <<= 1) {
#pragma unroll
    for (int d = sz >> 1; d > 0; d >>= 1) {
      if (d >= kE) {
        const int ld = d / kE;
        const bool lower = (lane & ld) == 0;
#pragma unroll
        for (int i = 0; i < kE; ++i) {
          const bool up = ((kE * lane + i) & sz) == 0;
          const double pk = __shfl_xor_sync(0xffffffffu, kv[i], ld);
          const int pi = __shfl_xor_sync(0xffffffffu, iv[i], ld);
          const bool mine_first = cand_before(kv[i], iv[i], pk, pi);
          if (!((lower == up) ? mine_first : !mine_first)) {
            kv[i] = pk;
            iv[i] = pi;
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < kE; ++i) {
          if (i & d) continue;
          const int j = i | d;
          const bool up = ((kE * lane + i) & sz) == 0;
          if (cand_before(kv[i], iv[i], kv[j], iv[j]) != up) {
            const double tk = kv[i];
            kv[i] = kv[j];
            kv[j] = tk;
            const int ti = iv[i];
            iv[i] = iv[j];
            iv[j] = ti;
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kE; ++i) {
    const int e = e0 + kE * lane + i;
    if (e < n) {
      key[e] = kv[i];
      idx[e] = iv[i];
    }
  }
}

template <int kT>
__global__ void __launch_bounds__(kT)
prefix_kernel(const float* __restrict__ z, const float* __restrict__ temps,
              const float* __restrict__ cost_tokens, const float* __restrict__ cost_ms, int n_pts,
              int staircase, int B, int K, int enable, const int32_t* budget_in,
              float* __restrict__ c_out, float* __restrict__ s_out,
              int32_t* __restrict__ verify_len, float* __restrict__ objective,
              int32_t* budget_out, unsigned* flags) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int n = B * K;
  // The merge buffers hold the keys themselves (survival, fp64) beside the
  // candidate ids k*B + b, so a comparison reads no index first.
  double* keyA = reinterpret_cast<double*>(smem_raw);  // [n]
  double* keyB = keyA + n;                              // [n]
  int* idxA = reinterpret_cast<int*>(keyB + n);         // [n]
  int* idxB = idxA + n;                                 // [n]
  int* lcount = idxB + n;                               // [B]
  __shared__ float s_xs[64], s_ys[64];
  __shared__ double shd[32];
  __shared__ int s_stop, s_budget;
  const int tid = threadIdx.x;

  if (tid == 0) {
    *flags = 0u;  // status of this call
    s_budget = budget_in != nullptr ? *budget_in : -1;  // read before budget_out is written
  }
  // cost table into shared memory; it must be ascending in tokens
  for (int i = tid; i < n_pts; i += kT) {
    s_xs[i] = cost_tokens[i];
    s_ys[i] = cost_ms[i];
  }
  __syncthreads();
  if (tid == 0) {
    bool ok = true;
    for (int i = 0; i + 1 < n_pts; ++i) ok = ok && (s_xs[i + 1] > s_xs[i]);
    if (!ok) raise_flag(flags, DSPARK_FLAG_BAD_TABLE);
    s_stop = n;
  }

  // c = sigmoid(z / T_k), one candidate per thread, in fp64
  for (int o = tid; o < n; o += kT) {
    const int k = o % K;
    const double ck = 1.0 / (1.0 + exp(-(double)z[o] / (double)temps[k]));
    c_out[o] = (float)ck;
    keyB[o] = ck;
  }
  for (int b = tid; b < B; b += kT) lcount[b] = 0;
  __syncthreads();
  // survival = running product over k: candidate (b, k) multiplies its
  // request's c values 0..k in order, the product a sequential loop forms,
  // so neighbouring threads write neighbouring words (one thread per
  // request, striding K words, met many-way bank conflicts).  Request b's
  // run of the merge is b * K .. b * K + K - 1, already in order.
  for (int o = tid; o < n; o += kT) {
    const int b = o / K, k = o - b * K;
    double run = 1.0;
    for (int j = 0; j <= k; ++j) run *= keyB[b * K + j];
    s_out[o] = (float)run;
    keyA[o] = run;
    idxA[o] = k * B + b;
  }
  __syncthreads();

  if (!enable) {
    double e = 0.0;
    for (int i = tid; i < n; i += kT) e += keyA[i];
    const double E = (double)B + block_sum_d<kT>(e, shd);
    for (int b = tid; b < B; b += kT) verify_len[b] = K;
    if (tid == 0) {
      const double t = cost_of(s_xs, s_ys, n_pts, staircase, (double)B + (double)n);
      if (!(t > 0.0)) raise_flag(flags, DSPARK_FLAG_BAD_TABLE);
      objective[0] = (float)(E / t);
      if (budget_out != nullptr) *budget_out = B + n;
    }
    return;
  }

  // blocks of kWarpSort candidates sorted by one warp each in registers
  // (the merge levels they replace, runs of K up to kWarpSort, cost about
  // 5 us each in shared memory), then a merge tree from runs of width
  // w = kWarpSort: each level merges pairs of neighbouring runs from
  // (skey, sidx) into (dkey, didx) (an unpaired last run is copied); the
  // heads of the two runs stay in registers
  // elements per lane: 8 where the register budget is 64 per thread (1024
  // threads), else 16
  constexpr int kE = kT >= 1024 ? 8 : 16;
  constexpr int kWarpSort = 32 * kE;
  for (int e0 = (tid >> 5) * kWarpSort; e0 < n; e0 += (kT >> 5) * kWarpSort)
    warp_sort<kE>(keyA, idxA, e0, n);
  __syncthreads();
  double* skey = keyA;
  int* sidx = idxA;
  double* dkey = keyB;
  int* didx = idxB;
  // outputs per thread and level; odd, so the lanes of a warp writing their
  // runs' k-th outputs (a stride of chunk elements) fall in different banks
  const int chunk = ((n + kT - 1) / kT) | 1;
  for (long long w = kWarpSort; w < n; w <<= 1) {
    const int o0 = min(tid * chunk, n), o1 = min(o0 + chunk, n);
    int i = 0, j = 0, a1 = 0, b1 = 0;  // cursors into the current pair's two runs
    double ka = 0.0, kb = 0.0;
    int ia = 0, ib = 0;
    int pair_end = -1;
    for (int o = o0; o < o1; ++o) {
      if (o >= pair_end) {
        // first output of this thread in a pair: merge-path split
        const long long p0 = (o / (2 * w)) * (2 * w);
        const int a0 = (int)p0;
        a1 = (int)min(p0 + w, (long long)n);
        const int b0 = a1;
        b1 = (int)min(p0 + 2 * w, (long long)n);
        pair_end = b1;
        const int q = o - a0;
        int lo = max(0, q - (b1 - b0)), hi = min(q, a1 - a0);
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          // does A[mid] come before B[q - mid - 1]?  then more of A is in
          const int x = a0 + mid, y = b0 + q - mid - 1;
          if (cand_before(skey[x], sidx[x], skey[y], sidx[y])) lo = mid + 1;
          else hi = mid;
        }
        i = a0 + lo;
        j = b0 + (q - lo);
        if (i < a1) { ka = skey[i]; ia = sidx[i]; }
        if (j < b1) { kb = skey[j]; ib = sidx[j]; }
      }
      if (j >= b1 || (i < a1 && cand_before(ka, ia, kb, ib))) {
        dkey[o] = ka;
        didx[o] = ia;
        if (++i < a1) { ka = skey[i]; ia = sidx[i]; }
      } else {
        dkey[o] = kb;
        didx[o] = ib;
        if (++j < b1) { kb = skey[j]; ib = sidx[j]; }
      }
    }
    __syncthreads();
    double* tk = skey;
    skey = dkey;
    dkey = tk;
    int* ti = sidx;
    sidx = didx;
    didx = ti;
  }
  const double* skeys = skey;  // survivals in order
  const int* idx = sidx;       // their candidate ids
  auto key = [&](int i) { return skeys[i]; };

  // E_i = B + sum of the first i survivals; each thread owns a contiguous run
  const int per = chunk;
  const int i0 = tid * per;
  double run = 0.0;
  for (int i = i0; i < i0 + per && i < n; ++i) run += key(i);
  double total;
  const double excl = block_excl_scan_d<kT>(run, shd, &total);
  // candidate i (0-based) raises the objective iff E_{i+1}/t(B+i+1) > E_i/t(B+i)
  double E = (double)B + excl;
  CostWalker cw{s_xs, s_ys, n_pts, staircase, 0};
  double t0 = (i0 < n) ? cw.at((double)B + (double)i0) : 1.0;
  for (int i = i0; i < i0 + per && i < n; ++i) {
    const double t1 = cw.at((double)B + (double)i + 1.0);
    const double E1 = E + key(i);
    if (!(t0 > 0.0) || !(t1 > 0.0)) raise_flag(flags, DSPARK_FLAG_BAD_TABLE);
    if (!(E1 / t1 > E / t0)) {
      atomicMin(&s_stop, i);
      break;
    }
    E = E1;
    t0 = t1;
  }
  __syncthreads();
  // the greedy cut, or the budget's (clamped to [0, n])
  int n_commit = s_stop;
  if (s_budget >= 0) {
    const long long want = (long long)s_budget - B;
    n_commit = want < 0 ? 0 : (want > n ? n : (int)want);
  }
  if (tid == 0 && budget_out != nullptr) *budget_out = B + s_stop;
  for (int i = tid; i < n_commit; i += kT) atomicAdd(&lcount[idx[i] % B], 1);
  __syncthreads();
  for (int b = tid; b < B; b += kT) verify_len[b] = lcount[b];
  // objective of the committed set: E at n_commit from the owning thread's run
  const bool owner = (n_commit == n) ? (tid == 0) : (n_commit >= i0 && n_commit < i0 + per);
  if (owner) {
    double Ec = (double)B + total;
    if (n_commit < n) {
      Ec = (double)B + excl;
      for (int i = i0; i < n_commit; ++i) Ec += key(i);
    }
    objective[0] = (float)(Ec / cost_of(s_xs, s_ys, n_pts, staircase, (double)B + (double)n_commit));
  }
}

}  // namespace dspark
