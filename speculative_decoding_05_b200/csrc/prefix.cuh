// prefix.cuh -- sequential temperature scaling, survival and the greedy
// hardware-aware prefix cut.
//
// The whole batch has at most kMaxCand = 8192 candidates (B*K), ordered by
// survival descending, ties by candidate index k*B + b ascending (position
// then request).  Survival never rises along a request's positions (each
// step multiplies by c in (0, 1]), so each request's K candidates are
// already a sorted run.  Two forms give the same order and outputs:
//  - one CTA (up to kPrefixSmallCand candidates, or the scheduler off):
//    blocks of 256 or 512 candidates are sorted by one warp each (a bitonic
//    network in registers and shuffles), then merged as a tree in shared
//    memory (each thread finds its output chunk's split by a merge-path
//    binary search, then merges it sequentially).  The buffers carry the
//    survival keys with the candidate ids: an earlier form that merged ids
//    and looked every key up by id spent 65 of its 86 us at the stress
//    shape in the merge.
//  - many CTAs (more candidates): each places a slice of at most 63
//    candidates in the order by counting, for every candidate, how many
//    slice members precede it (see prefix_rank_kernel); the last CTA runs
//    the scan.
// The expected-emitted-token prefix sums are a block scan in fp64, and the
// early stop is the first index where E/t(N) does not increase.
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

// Arguments of the prefix-cut kernels (device pointers; see the C entry
// dspark_confidence_prefix_async).
struct PrefixArgs {
  const float* z;
  const float* temps;
  const float* cost_tokens;
  const float* cost_ms;
  int n_pts, staircase, B, K, enable;
  const int32_t* budget_in;
  float* c_out;
  float* s_out;
  int32_t* verify_len;
  float* objective;
  int32_t* budget_out;
  unsigned* flags;
};

// The cost table into shared memory (thread 0 checks that it ascends), the
// budget of this call (read before any budget_out write) and the stop index
// preset to n.  Contains one barrier.
template <int kT>
__device__ __forceinline__ void prefix_setup(const PrefixArgs& a, float* s_xs, float* s_ys,
                                             int* s_budget, int* s_stop, int n) {
  for (int i = threadIdx.x; i < a.n_pts; i += kT) {
    s_xs[i] = a.cost_tokens[i];
    s_ys[i] = a.cost_ms[i];
  }
  if (threadIdx.x == 0) *s_budget = a.budget_in != nullptr ? *a.budget_in : -1;
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    for (int i = 0; i + 1 < a.n_pts; ++i) ok = ok && (s_xs[i + 1] > s_xs[i]);
    if (!ok) raise_flag(a.flags, DSPARK_FLAG_BAD_TABLE);
    *s_stop = n;
  }
}

// The greedy scan and the commit over the candidates in order (survivals
// skeys, candidate ids idx = k*B + b), in one CTA of kT threads.  lcount
// [B] must be zero and every input visible to the block on entry.
template <int kT>
__device__ __forceinline__ void prefix_cut(const PrefixArgs& a, const double* skeys,
                                           const int* idx, int* lcount, const float* s_xs,
                                           const float* s_ys, int budget, int* s_stop,
                                           double* shd) {
  const int B = a.B, n = a.B * a.K, tid = threadIdx.x;
  // E_i = B + sum of the first i survivals; each thread owns a contiguous run
  const int per = ((n + kT - 1) / kT) | 1;
  const int i0 = tid * per;
  double run = 0.0;
  for (int i = i0; i < i0 + per && i < n; ++i) run += skeys[i];
  double total;
  const double excl = block_excl_scan_d<kT>(run, shd, &total);
  // candidate i (0-based) raises the objective iff E_{i+1}/t(B+i+1) >
  // E_i/t(B+i); the right side is the left side of the step before
  double E = (double)B + excl;
  CostWalker cw{s_xs, s_ys, a.n_pts, a.staircase, 0};
  double t0 = (i0 < n) ? cw.at((double)B + (double)i0) : 1.0;
  double obj0 = E / t0;
  for (int i = i0; i < i0 + per && i < n; ++i) {
    const double t1 = cw.at((double)B + (double)i + 1.0);
    const double E1 = E + skeys[i];
    if (!(t0 > 0.0) || !(t1 > 0.0)) raise_flag(a.flags, DSPARK_FLAG_BAD_TABLE);
    const double obj1 = E1 / t1;
    if (!(obj1 > obj0)) {
      atomicMin(s_stop, i);
      break;
    }
    E = E1;
    t0 = t1;
    obj0 = obj1;
  }
  __syncthreads();
  // the greedy cut, or the budget's (clamped to [0, n])
  const int stop = *s_stop;
  int n_commit = stop;
  if (budget >= 0) {
    const long long want = (long long)budget - B;
    n_commit = want < 0 ? 0 : (want > n ? n : (int)want);
  }
  if (tid == 0 && a.budget_out != nullptr) *a.budget_out = B + stop;
  for (int i = tid; i < n_commit; i += kT) {
    const int id = idx[i];
    if ((unsigned)id < (unsigned)n) atomicAdd(&lcount[id % B], 1);
  }
  __syncthreads();
  for (int b = tid; b < B; b += kT) a.verify_len[b] = lcount[b];
  // objective of the committed set: E at n_commit from the owning thread's run
  const bool owner = (n_commit == n) ? (tid == 0) : (n_commit >= i0 && n_commit < i0 + per);
  if (owner) {
    double Ec = (double)B + total;
    if (n_commit < n) {
      Ec = (double)B + excl;
      for (int i = i0; i < n_commit; ++i) Ec += skeys[i];
    }
    a.objective[0] =
        (float)(Ec / cost_of(s_xs, s_ys, a.n_pts, a.staircase, (double)B + (double)n_commit));
  }
}

// Single-CTA form: every step in one block (the form for up to
// kPrefixSmallCand candidates, and for enable == 0).
template <int kT>
__global__ void __launch_bounds__(kT) prefix_kernel(const PrefixArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int B = a.B, K = a.K, n = B * K;
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

  if (tid == 0) *a.flags = 0u;  // status of this call
  prefix_setup<kT>(a, s_xs, s_ys, &s_budget, &s_stop, n);

  // c = sigmoid(z / T_k), one candidate per thread, in fp64
  for (int o = tid; o < n; o += kT) {
    const int k = o % K;
    const double ck = 1.0 / (1.0 + exp(-(double)a.z[o] / (double)a.temps[k]));
    a.c_out[o] = (float)ck;
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
    a.s_out[o] = (float)run;
    keyA[o] = run;
    idxA[o] = k * B + b;
  }
  __syncthreads();

  if (!a.enable) {
    double e = 0.0;
    for (int i = tid; i < n; i += kT) e += keyA[i];
    const double E = (double)B + block_sum_d<kT>(e, shd);
    for (int b = tid; b < B; b += kT) a.verify_len[b] = K;
    if (tid == 0) {
      const double t = cost_of(s_xs, s_ys, a.n_pts, a.staircase, (double)B + (double)n);
      if (!(t > 0.0)) raise_flag(a.flags, DSPARK_FLAG_BAD_TABLE);
      a.objective[0] = (float)(E / t);
      if (a.budget_out != nullptr) *a.budget_out = B + n;
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
  prefix_cut<kT>(a, skey, sidx, lcount, s_xs, s_ys, s_budget, &s_stop, shd);
}

// ---------------------------------------------------------------------------
// Multi-CTA form (more than kPrefixSmallCand candidates, scheduler on)
// ---------------------------------------------------------------------------
//
// The single CTA above is bound by one SM's issue rate (about 70 us for
// 8192 candidates, most of it in the sort).  This form spreads the order
// over the GPU:
//   1. prefix_surv_kernel: c and survival exactly as prefix_kernel forms
//      them, each CTA over whole requests; the fp64 survivals go to the
//      workspace indexed by candidate id k*B + b.
//   2. prefix_rank_kernel: CTA j takes the candidates with ids in
//      [j n / G, (j+1) n / G) (at most kRankSlice) as its slice and sorts
//      them in one warp.  For every candidate e of the batch, q(e) = the
//      number of slice members that come before e (a binary search in
//      shared memory).  e comes before slice member p exactly when
//      q(e) <= p (e not p itself), so with h[q] = #{e : q(e) = q}, member p
//      has h[0] + ... + h[p] - 1 candidates before it: its place in the
//      order.  Each CTA writes its members' (survival, id) there; the last
//      CTA to finish (a counter) reads the whole order back and runs
//      prefix_cut, the same greedy scan as the single-CTA form.
// The order is the same strict total order (a NaN survival ranks as -1,
// after every real one, so the places stay a permutation), hence the same
// outputs.

constexpr int kSurvThreads = 256;
constexpr int kRankThreads = kPrefixThreads;
constexpr int kRankSlice = 63;  // slice members per CTA; slot 63 stays a sentinel
constexpr int kRankPer = kMaxCand / kRankThreads;  // candidates per thread in the count
// the rank pass's counter sits in the workspace header, after the status word
constexpr size_t kPrefixCounterOff = 128;

__device__ __forceinline__ double rank_key(double s) { return s == s ? s : -1.0; }

__global__ void __launch_bounds__(kSurvThreads)
prefix_surv_kernel(const PrefixArgs a, double* __restrict__ surv_id, unsigned* counter) {
  extern __shared__ double s_c[];  // c of this CTA's requests
  // the rank pass may be scheduled now; it waits for this grid to complete
  grid_dep_launch();
  const int B = a.B, K = a.K;
  const int rb = max(1, kSurvThreads / K);  // requests per CTA
  const int b0 = blockIdx.x * rb, nb = min(rb, B - b0);
  const int m = nb * K;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *a.flags = 0u;  // status of this call
    *counter = 0u;
  }
  for (int l = threadIdx.x; l < m; l += kSurvThreads) {
    const int o = b0 * K + l, k = l % K;
    const double ck = 1.0 / (1.0 + exp(-(double)a.z[o] / (double)a.temps[k]));
    a.c_out[o] = (float)ck;
    s_c[l] = ck;
  }
  __syncthreads();
  for (int l = threadIdx.x; l < m; l += kSurvThreads) {
    const int bl = l / K, k = l - bl * K;
    double run = 1.0;
    for (int j = 0; j <= k; ++j) run *= s_c[bl * K + j];
    a.s_out[b0 * K + l] = (float)run;
    surv_id[(size_t)k * B + b0 + bl] = run;
  }
}

__global__ void __launch_bounds__(kRankThreads, 1)
prefix_rank_kernel(const PrefixArgs a, const double* surv_id, double* okey, int* oidx,
                   unsigned* counter) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ double sl_key[64];
  __shared__ int sl_id[64];
  __shared__ int hist[64];
  __shared__ int s_last;
  __shared__ float s_xs[64], s_ys[64];
  __shared__ double shd[32];
  __shared__ int s_stop, s_budget;
  const int B = a.B, n = a.B * a.K, tid = threadIdx.x, lane = tid & 31;
  const int G = gridDim.x;
  const int p0 = (int)((long long)blockIdx.x * n / G);
  const int P = (int)((long long)(blockIdx.x + 1) * n / G) - p0;  // 1..kRankSlice
  if (tid < 64) hist[tid] = 0;
  // Every read of the survival pass's output comes after this wait, as a
  // volatile load (__ldcg) that the compiler keeps behind it: an ordinary
  // load of read-only data may be issued before the wait and return what
  // the workspace held before the survival pass wrote it.
  grid_dep_wait();
  // this thread's candidates: ids tid, tid + kRankThreads, ...
  double ek[kRankPer];
#pragma unroll
  for (int j = 0; j < kRankPer; ++j) {
    const int e = tid + j * kRankThreads;
    ek[j] = e < n ? rank_key(__ldcg(surv_id + e)) : 0.0;
  }
  if (tid < 32) {
    // the slice, sorted by one warp; slots past P are sentinels that come
    // before no candidate
    for (int p = lane; p < 64; p += 32) {
      sl_key[p] = p < P ? rank_key(__ldcg(surv_id + p0 + p)) : -CUDART_INF;
      sl_id[p] = p < P ? p0 + p : 0x7fffffff;
    }
    __syncwarp();
    warp_sort<2>(sl_key, sl_id, 0, P);
  }
  __syncthreads();
  // q(e) by binary lifting over the 64 slots (q <= P <= 63)
#pragma unroll
  for (int j = 0; j < kRankPer; ++j) {
    const int e = tid + j * kRankThreads;
    const bool valid = e < n;
    int q = 0;
#pragma unroll
    for (int step = 32; step > 0; step >>= 1) {
      const int t = q + step - 1;
      if (cand_before(sl_key[t], sl_id[t], ek[j], e)) q += step;
    }
    // most candidates fall before or after the whole slice: those before
    // are counted per warp, those after are not needed
    const unsigned m0 = __ballot_sync(0xffffffffu, valid && q == 0);
    if (lane == 0 && m0 != 0u) atomicAdd(&hist[0], __popc(m0));
    if (valid && q > 0 && q < P) atomicAdd(&hist[q], 1);
  }
  __syncthreads();
  if (tid < 32) {
    // place of member p = h[0] + ... + h[p] - 1 (lane l holds p = 2l, 2l+1)
    const int pa = 2 * lane, pb = pa + 1;
    const int ha = pa < P ? hist[pa] : 0, hb = pb < P ? hist[pb] : 0;
    int incl = ha + hb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - ha - hb;
    if (pa < P) {
      const int r = min(max(excl + ha - 1, 0), n - 1);
      okey[r] = __ldcg(surv_id + sl_id[pa]);
      oidx[r] = sl_id[pa];
    }
    if (pb < P) {
      const int r = min(max(excl + ha + hb - 1, 0), n - 1);
      okey[r] = __ldcg(surv_id + sl_id[pb]);
      oidx[r] = sl_id[pb];
    }
  }
  // the last CTA to get here runs the scan over the whole order
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(counter, 1u) == (unsigned)(G - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  double* skeys = reinterpret_cast<double*>(smem_raw);  // [n]
  int* sidx = reinterpret_cast<int*>(skeys + n);        // [n]
  int* lcount = sidx + n;                               // [B]
  for (int i = tid; i < n; i += kRankThreads) {
    skeys[i] = __ldcg(okey + i);
    sidx[i] = __ldcg(oidx + i);
  }
  for (int b = tid; b < B; b += kRankThreads) lcount[b] = 0;
  prefix_setup<kRankThreads>(a, s_xs, s_ys, &s_budget, &s_stop, n);
  prefix_cut<kRankThreads>(a, skeys, sidx, lcount, s_xs, s_ys, s_budget, &s_stop, shd);
}

// Workspace of the prefix cut: the header, then (multi-CTA form) the
// survivals by candidate id and the order's keys and ids.
inline bool prefix_multi(int n, int enable) { return enable && n > kPrefixSmallCand; }
inline size_t prefix_ws_bytes(int n) {
  return kHeaderBytes + align256((size_t)n * 8) * 2 + align256((size_t)n * 4);
}

}  // namespace dspark
