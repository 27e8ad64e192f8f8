// sample.cuh -- two-level inverse-CDF sampling over chunk partials.
//
// The projection kernels leave one (reference max, partial sum) pair per
// 32-row chunk of the vocabulary.  A sampler CTA (one per request) turns
// them into chunk weights, scans them in fp64 to find the chunk where the
// running mass first exceeds u * Z, then re-computes the 32 weights of
// that chunk exactly and scans them (fp64) to find the token.
#pragma once

#include "proj_simt.cuh"

namespace dspark {

constexpr int kSampleThreads = 256;
constexpr int kMaxRank = 1024;  // largest r the samplers stage in shared memory

struct ChunkPick {
  int chunk;      // chosen chunk
  double before;  // running mass before the chunk
  double total;   // Z
  double target;  // u * Z
};

// Scan chunk weights w(c) >= 0 in vocabulary order and pick the chunk whose
// running sum first exceeds u * Z.  Every thread owns a contiguous range of
// chunks.  If rounding leaves no crossing, the last chunk with positive
// weight is taken.  Result valid in every thread after the call.
template <class WFn>
__device__ ChunkPick pick_chunk(int n_chunks, double u, WFn wfn) {
  __shared__ double sh[32];
  __shared__ double s_start[kSampleThreads + 1];
  __shared__ int s_chunk, s_last;
  __shared__ double s_before;
  const int per = (n_chunks + kSampleThreads - 1) / kSampleThreads;
  const int c0 = min(threadIdx.x * per, n_chunks);
  const int c1 = min(c0 + per, n_chunks);
  double sum = 0.0;
  int last_pos = -1;
  for (int c = c0; c < c1; ++c) {
    const double w = wfn(c);
    sum += w;
    if (w > 0.0) last_pos = c;
  }
  double total;
  const double excl = block_excl_scan_d<kSampleThreads>(sum, sh, &total);
  s_start[threadIdx.x] = excl;
  if (threadIdx.x == 0) {
    s_start[kSampleThreads] = total;
    s_chunk = -1;
    s_last = -1;
  }
  __syncthreads();
  const double target = u * total;
  if (last_pos >= 0) atomicMax(&s_last, last_pos);
  // The thread intervals [start_t, start_{t+1}) partition [0, total), so
  // exactly one thread owns the target when 0 <= target < total.
  const double end = s_start[threadIdx.x + 1];
  if (excl <= target && target < end) {
    double cum = excl;
    int pick = -1, lastp = -1;
    double before = excl, before_last = excl;
    for (int c = c0; c < c1; ++c) {
      const double w = wfn(c);
      const double nxt = cum + w;
      if (w > 0.0) {
        lastp = c;
        before_last = cum;
      }
      if (nxt > target && w > 0.0) {
        pick = c;
        before = cum;
        break;
      }
      cum = nxt;
    }
    if (pick < 0) {
      pick = lastp;
      before = before_last;
    }
    if (pick >= 0) {
      s_chunk = pick;
      s_before = before;
    }
  }
  __syncthreads();
  ChunkPick p;
  p.total = total;
  p.target = target;
  if (s_chunk >= 0) {
    p.chunk = s_chunk;
    p.before = s_before;
  } else {
    // no crossing (u*Z rounded up to Z): the last chunk with positive weight,
    // and the element scan then takes its last positive entry.
    p.chunk = s_last >= 0 ? s_last : 0;
    p.before = -CUDART_INF;
  }
  return p;
}

// Element scan inside the chosen chunk (called by one full warp): e = this
// lane's weight (0 for rows past V).  Returns the chosen lane: the first
// whose running sum exceeds the target, else the last with positive weight,
// else lane 0.
__device__ __forceinline__ int pick_lane(double e, double before, double target) {
  const double cum = before + warp_incl_scan_d(e);
  const unsigned hit = __ballot_sync(0xffffffffu, cum > target && e > 0.0);
  if (hit) return __ffs(hit) - 1;
  const unsigned pos = __ballot_sync(0xffffffffu, e > 0.0);
  if (pos) return 31 - __clz(pos);
  return 0;
}

// Draft sampler for position k: one CTA per request.
template <typename TW>
__global__ void __launch_bounds__(kSampleThreads)
draft_sample_kernel(const float* __restrict__ base, const TW* __restrict__ U,
                    const TW* __restrict__ W, int V, int r, int K, int k,
                    const int32_t* __restrict__ prev_token, int32_t* __restrict__ tokens,
                    const float* __restrict__ inv_temp, const float* __restrict__ u_draft,
                    const float2* __restrict__ part, int n_chunks,
                    const float* __restrict__ draft_bias, float* __restrict__ p_tok,
                    float* __restrict__ lse, float* __restrict__ ref_max,
                    float* __restrict__ ref_sum, unsigned* flags) {
  __shared__ __align__(16) float u_s[kMaxRank];
  __shared__ float shf[32];
  const int b = blockIdx.x;
  const float it = checked_inv_temp(inv_temp, b, flags);
  const float it2 = it * kLog2e;
  const float2* pb = part + (size_t)b * n_chunks;

  float m = -CUDART_INF_F;
  for (int c = threadIdx.x; c < n_chunks; c += kSampleThreads) m = fmaxf(m, pb[c].x);
  const float M = block_max<kSampleThreads>(m, shf);

  const double u = (double)u_draft[(size_t)b * K + k];
  ChunkPick pk = pick_chunk(n_chunks, u, [&](int c) -> double {
    const float2 p = pb[c];
    return (double)(p.y * ex2((p.x - M) * it2));
  });

  int xp = (k == 0) ? prev_token[b] : tokens[(size_t)b * K + (k - 1)];
  xp = checked_token(xp, V, k == 0, flags);
  if (xp >= 0 && draft_bias == nullptr)
    for (int i = threadIdx.x; i < r; i += kSampleThreads) u_s[i] = to_f32(U[(size_t)xp * r + i]);
  __syncthreads();

  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int v = pk.chunk * kChunk + lane;
    const bool valid = v < V;
    float e = 0.0f;
    if (valid) {
      const size_t row = ((size_t)b * K + k) * (size_t)V;
      const float bias = draft_bias != nullptr ? draft_bias[row + v]
                         : (xp >= 0)           ? dot_row(W + (size_t)v * r, u_s, r)
                                               : 0.0f;
      const float bv = base[row + v];
      e = ex2(((bv - M) + bias) * it2);
    }
    const int pick = pick_lane(valid ? (double)e : 0.0, pk.before, pk.target);
    if (lane == pick) {
      const double Z = pk.total;
      const size_t o = (size_t)b * K + k;
      if (!(Z > 0.0) || !isfinite(Z)) {
        raise_flag(flags, DSPARK_FLAG_NONFINITE);
        tokens[o] = 0;
        p_tok[o] = 0.0f;
        lse[o] = CUDART_NAN_F;
        ref_max[o] = M;
        ref_sum[o] = 1.0f;
      } else {
        tokens[o] = valid ? v : 0;
        p_tok[o] = (float)((double)e / Z);
        lse[o] = (float)((double)M * (double)it + log(Z));
        ref_max[o] = M;
        ref_sum[o] = (float)Z;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Two-level draft sampler of the tensor-core projection: one warp per request
// ---------------------------------------------------------------------------
//
// The projection's CTA (bb, pi) covers the contiguous tile range
// [pi * n_tiles / n_ctas, (pi + 1) * n_tiles / n_ctas) for the requests of
// block bb; its two epilogue warpgroups each leave one partial per request
// (warpgroup g: the chunks 4t + 2g, 4t + 2g + 1 of its tiles).  Per request
// the sampler
//   1. merges each CTA's two partials into the weight of its range and
//      scans the CTA weights in vocabulary order (fp64) to find the CTA
//      whose range holds u * Z;
//   2. scans that CTA's chunk partials (vocabulary order, fp64);
//   3. re-computes the 32 weights of the chosen chunk and scans them.
// The decisions are those of the one-level scan over all chunks up to
// float rounding of the partial sums (about 1e-7 relative).
// Requests (one warp each) per CTA: the sampler is a chain of dependent
// loads per request, and spreading the requests over more SMs shortened the
// draft call by 2 % at B = 512 and 7 % at B = 64 against 8 warps a CTA.
constexpr int kS2Warps = 2;
constexpr int kS2Parts = 2;  // partials per CTA and request (epilogue warpgroups)

// Weight of a softmax partial (A, s) relative to the reference max M:
// s * 2^((A - M) * it2), 0 for an empty partial.
__device__ __forceinline__ double partial_weight(float2 q, float M, float it2) {
  return (q.x == -CUDART_INF_F) ? 0.0 : (double)(q.y * ex2((q.x - M) * it2));
}

__device__ __forceinline__ double cta_weight(const float2* q, float M, float it2) {
  double w = 0.0;
#pragma unroll
  for (int g = 0; g < kS2Parts; ++g) w += partial_weight(q[g], M, it2);
  return w;
}

// Warp-wide scan of n items in order, weights wfn(i) >= 0: lane l owns the
// contiguous run [l * per, (l + 1) * per) and its running sum.  warp_total
// and warp_pick associate the sum identically.
template <class WFn>
__device__ __forceinline__ double warp_run_sum(int n, WFn wfn, int* i0, int* i1, int* last_pos) {
  const int lane = threadIdx.x & 31;
  const int per = (n + 31) / 32;
  *i0 = min(lane * per, n);
  *i1 = min(*i0 + per, n);
  double sum = 0.0;
  *last_pos = -1;
  for (int i = *i0; i < *i1; ++i) {
    const double w = wfn(i);
    sum += w;
    if (w > 0.0) *last_pos = i;
  }
  return sum;
}

template <class WFn>
__device__ __forceinline__ double warp_total(int n, WFn wfn) {
  int i0, i1, lp;
  const double sum = warp_run_sum(n, wfn, &i0, &i1, &lp);
  return __shfl_sync(0xffffffffu, warp_incl_scan_d(sum), 31);
}

// The item whose interval [before, before + w) holds `target`, the items'
// intervals laid end to end from `base`; *before is set.  If rounding
// leaves no crossing, the last item with positive weight and *before =
// -inf (the element scan then takes its last positive entry).
template <class WFn>
__device__ __forceinline__ int warp_pick(int n, double base, double target, WFn wfn,
                                         double* before) {
  const int lane = threadIdx.x & 31;
  int i0, i1, last_pos;
  const double sum = warp_run_sum(n, wfn, &i0, &i1, &last_pos);
  const double incl = warp_incl_scan_d(sum);
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  // lane intervals [base + excl, base + incl) partition [base, base + total)
  const bool mine = sum > 0.0 && base + excl <= target && target < base + incl;
  int pick = -1;
  double bef = 0.0;
  if (mine) {
    double cum = base + excl;
    for (int i = i0; i < i1; ++i) {
      const double w = wfn(i);
      if (w > 0.0 && cum + w > target) {
        pick = i;
        bef = cum;
        break;
      }
      cum += w;
    }
  }
  const unsigned own = __ballot_sync(0xffffffffu, pick >= 0);
  if (own) {
    const int src = __ffs(own) - 1;
    *before = __shfl_sync(0xffffffffu, bef, src);
    return __shfl_sync(0xffffffffu, pick, src);
  }
  const unsigned pos = __ballot_sync(0xffffffffu, last_pos >= 0);
  *before = -CUDART_INF;
  if (!pos) return 0;
  return __shfl_sync(0xffffffffu, last_pos, 31 - __clz(pos));
}

template <typename TW>
__global__ void __launch_bounds__(kS2Warps * 32)
draft_sample2_kernel(const float* __restrict__ base, const TW* __restrict__ U,
                     const TW* __restrict__ W, int V, int r, int B, int K, int k,
                     const int32_t* __restrict__ prev_token, int32_t* __restrict__ tokens,
                     const float* __restrict__ inv_temp, const float* __restrict__ u_draft,
                     const float2* __restrict__ part, int n_chunks,
                     const float2* __restrict__ cta_part, int n_ctas, int n_tiles,
                     const float* __restrict__ draft_bias, float* __restrict__ p_tok,
                     float* __restrict__ lse, float* __restrict__ ref_max,
                     float* __restrict__ ref_sum, unsigned* flags,
                     const float* __restrict__ state = nullptr) {
  // state [B, r] fp32 (RNN head): the re-computed bias is state[b] . W[v]
  // instead of U[x_prev] . W[v]
  __shared__ __align__(16) float u_s[kS2Warps][kMaxRank];
  // the next position's projection may begin launching now (it waits for
  // this kernel before it touches anything this kernel reads or writes).
  // This kernel itself is a plain launch: launching it behind the
  // projection with a dependency as well measured 10 % slower on the draft.
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * kS2Warps + warp;
  if (b >= B) return;  // whole warps only; no block-wide synchronisation follows
  const float it = checked_inv_temp(inv_temp, b, flags);
  const float it2 = it * kLog2e;
  int xp = (k == 0) ? prev_token[b] : tokens[(size_t)b * K + (k - 1)];
  xp = checked_token(xp, V, k == 0, flags);
  float* us = u_s[warp];
  if (state != nullptr) {
    xp = 0;  // the state always contributes a bias
    if (draft_bias == nullptr)
      for (int i = lane; i < r; i += 32) us[i] = state[(size_t)b * r + i];
  } else if (xp >= 0 && draft_bias == nullptr) {
    for (int i = lane; i < r; i += 32) us[i] = to_f32(U[(size_t)xp * r + i]);
  }

  // level 1: the CTAs of this request's block, in vocabulary order
  const float2* cp = cta_part + (size_t)b * n_ctas * kS2Parts;
  float m = -CUDART_INF_F;
  for (int i = lane; i < n_ctas * kS2Parts; i += 32) m = fmaxf(m, cp[i].x);
  const float M = warp_max(m);
  auto wcta = [&](int i) { return cta_weight(cp + i * kS2Parts, M, it2); };
  const double Z = warp_total(n_ctas, wcta);
  const double target = (double)u_draft[(size_t)b * K + k] * Z;
  double before1;
  const int cta = warp_pick(n_ctas, 0.0, target, wcta, &before1);

  // level 2: the chunks of that CTA's tile range
  const int t0 = (int)((long long)cta * n_tiles / n_ctas);
  const int t1 = (int)((long long)(cta + 1) * n_tiles / n_ctas);
  const int ch0 = t0 * 4, ch1 = min(t1 * 4, n_chunks);
  const float2* pb = part + (size_t)b * n_chunks;
  double before2;
  const int chunk = ch0 + warp_pick(
      max(ch1 - ch0, 0), before1, target,
      [&](int i) { return partial_weight(pb[ch0 + i], M, it2); }, &before2);

  // level 3: the 32 rows of the chosen chunk
  __syncwarp();
  const int v = chunk * kChunk + lane;
  const bool valid = v < V;
  float e = 0.0f;
  const size_t row = ((size_t)b * K + k) * (size_t)V;
  if (valid) {
    const float bias = draft_bias != nullptr ? draft_bias[row + v]
                       : (xp >= 0)           ? dot_row(W + (size_t)v * r, us, r)
                                             : 0.0f;
    e = ex2(((base[row + v] - M) + bias) * it2);
  }
  const int pick = pick_lane(valid ? (double)e : 0.0, before2, target);
  if (lane == pick) {
    const size_t o = (size_t)b * K + k;
    if (!(Z > 0.0) || !isfinite(Z)) {
      raise_flag(flags, DSPARK_FLAG_NONFINITE);
      tokens[o] = 0;
      p_tok[o] = 0.0f;
      lse[o] = CUDART_NAN_F;
      ref_max[o] = M;
      ref_sum[o] = 1.0f;
    } else {
      tokens[o] = valid ? v : 0;
      p_tok[o] = (float)((double)e / Z);
      lse[o] = (float)((double)M * (double)it + log(Z));
      ref_max[o] = M;
      ref_sum[o] = (float)Z;
    }
  }
}

// Correction / bonus sampler: one CTA per request.  Draws from the residual
// max(0, p_t - p_d) (or p_t for a bonus draw); falls back to p_t when the
// residual mass is zero.
template <typename TW>
__global__ void __launch_bounds__(kSampleThreads)
residual_sample_kernel(const float* __restrict__ target, const float* __restrict__ base,
                       const TW* __restrict__ U, const TW* __restrict__ W, int V, int r, int K,
                       const float* __restrict__ inv_temp, const float* __restrict__ u_res,
                       const ResInfo* __restrict__ info, const float2* __restrict__ rpart,
                       int n_chunks, const float* __restrict__ draft_bias,
                       int32_t* __restrict__ out_tokens,
                       int32_t* __restrict__ last_token, unsigned* flags) {
  __shared__ __align__(16) float u_s[kMaxRank];
  __shared__ double shd[32];
  const int b = blockIdx.x;
  const ResInfo ri = info[b];
  const float it2 = checked_inv_temp(inv_temp, b, flags) * kLog2e;
  const float2* pb = rpart + (size_t)b * n_chunks;

  double q = 0.0;
  for (int c = threadIdx.x; c < n_chunks; c += kSampleThreads) q += (double)pb[c].x;
  const double Qtot = block_sum_d<kSampleThreads>(q, shd);
  const bool use_q = Qtot > 0.0 && isfinite(Qtot);

  const double u = (double)u_res[b];
  ChunkPick pk = pick_chunk(n_chunks, u, [&](int c) -> double {
    const float2 p = pb[c];
    return (double)(use_q ? p.x : p.y);
  });

  const int xp = ri.bonus ? -1 : ri.x_prev;
  if (xp >= 0 && draft_bias == nullptr)
    for (int i = threadIdx.x; i < r; i += kSampleThreads) u_s[i] = to_f32(U[(size_t)xp * r + i]);
  __syncthreads();

  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int v = pk.chunk * kChunk + lane;
    const bool valid = v < V;
    double e = 0.0;
    if (valid) {
      const size_t drow = ((size_t)b * K + (ri.bonus ? 0 : ri.j)) * (size_t)V;
      float bias = 0.0f;
      if (!ri.bonus) {
        if (draft_bias != nullptr) bias = draft_bias[drow + v];
        else if (xp >= 0) bias = dot_row(W + (size_t)v * r, u_s, r);
      }
      const float t = target[(size_t)ri.row * V + v];
      const float bv = ri.bonus ? 0.0f : base[drow + v];
      float pt;
      const float qv = residual_q(t, bv, bias, ri, it2, &pt);
      e = (double)(use_q ? qv : pt);
    }
    const int pick = pick_lane(e, pk.before, pk.target);
    if (lane == pick) {
      if (!(pk.total > 0.0) || !isfinite(pk.total)) raise_flag(flags, DSPARK_FLAG_NONFINITE);
      const int tok = valid ? v : 0;
      out_tokens[(size_t)b * (K + 1) + ri.j] = tok;
      if (last_token != nullptr) last_token[b] = tok;
    }
  }
}

}  // namespace dspark
