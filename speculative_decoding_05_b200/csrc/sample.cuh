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
  // The next position's projection is launched behind this kernel with a
  // programmatic dependency; let it start its prologue once this kernel is
  // running (the wait is a no-op for a plain launch).
  grid_dep_wait();
  grid_dep_launch();
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
