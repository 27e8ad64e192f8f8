// verify.cuh -- target-row statistics and the accept scan of the
// rejection-sampling verify.
#pragma once

#include "proj_simt.cuh"

namespace dspark {

constexpr int kStatsThreads = 256;  // kSeg / kStatsThreads = 32 elements per thread

// Clamped verify length of request b (a value outside [0, K] raises
// DSPARK_FLAG_BAD_LENGTH and is clamped).
__device__ __forceinline__ int checked_len(const int32_t* verify_len, int b, int K, unsigned* flags) {
  int L = verify_len[b];
  if (L < 0 || L > K) {
    raise_flag(flags, DSPARK_FLAG_BAD_LENGTH);
    L = L < 0 ? 0 : K;
  }
  return L;
}

// Target row of request b, position p; a row outside [0, n_rows) raises
// DSPARK_FLAG_BAD_LENGTH and is clamped.
__device__ __forceinline__ long long checked_row(const int64_t* row_start, int b, int p,
                                                 long long n_rows, unsigned* flags) {
  long long row = (long long)row_start[b] + p;
  if (row < 0 || row >= n_rows) {
    raise_flag(flags, DSPARK_FLAG_BAD_LENGTH);
    row = row < 0 ? 0 : n_rows - 1;
  }
  return row;
}

// Softmax statistics of the verified target rows, split over the
// vocabulary: grid (n_segs, B*(K+1)); CTA (seg, b*(K+1)+p) reduces
// elements [seg*kSeg, (seg+1)*kSeg) of the row of (b, p) when p <= L_b to
// (max t, sum exp((t - max) * inv_temp)).  Target logits are streamed with
// 128-bit evict-first loads (they are read once).
__global__ void __launch_bounds__(kStatsThreads)
target_stats_kernel(const float* __restrict__ target, long long n_rows,
                    const int64_t* __restrict__ row_start, const int32_t* __restrict__ verify_len,
                    const float* __restrict__ inv_temp, int V, int K, float2* __restrict__ tpart,
                    int n_segs, unsigned* flags) {
  __shared__ float shf[32];
  __shared__ double shd[32];
  const int rid = blockIdx.y;
  const int b = rid / (K + 1), p = rid % (K + 1);
  const int L = checked_len(verify_len, b, K, flags);
  if (p > L) return;
  const long long row = checked_row(row_start, b, p, n_rows, flags);
  const float it2 = checked_inv_temp(inv_temp, b, flags) * kLog2e;
  const float* trow = target + (size_t)row * V;
  const int seg = blockIdx.x;
  const int e0 = seg * kSeg;

  constexpr int kVec = kSeg / (4 * kStatsThreads);  // float4 per thread
  const uint64_t pol = policy_evict_first();
  float4 x[kVec];
  float m = -CUDART_INF_F;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int e = e0 + (i * kStatsThreads + threadIdx.x) * 4;
    if (e < V) {  // V % 4 == 0: a float4 is either fully inside or outside
      x[i] = ld_stream4(trow + e, pol);
      m = fmaxf(m, fmaxf(fmaxf(x[i].x, x[i].y), fmaxf(x[i].z, x[i].w)));
    } else {
      x[i] = make_float4(-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F);
    }
  }
  const float M = block_max<kStatsThreads>(m, shf);
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int e = e0 + (i * kStatsThreads + threadIdx.x) * 4;
    if (e < V) {
      s += ex2((x[i].x - M) * it2) + ex2((x[i].y - M) * it2) + ex2((x[i].z - M) * it2) +
           ex2((x[i].w - M) * it2);
    }
  }
  const double S = block_sum_d<kStatsThreads>((double)s, shd);
  if (threadIdx.x == 0) tpart[(size_t)rid * n_segs + seg] = make_float2(M, (float)S);
}

// Accept scan: one warp per request.  Lane p handles verified row p
// (p <= L_b, looping by 32 for K >= 32): combines the row's segment
// statistics, and for p < L_b evaluates u_acc < p_t(x_p) / p_d(x_p).
// n_acc = first rejected position (or L_b).  Writes n_accepted, the
// accepted tokens and -1 padding of out_tokens, and the ResInfo of the
// correction / bonus row.
__global__ void __launch_bounds__(128)
accept_kernel(const float* __restrict__ target, long long n_rows,
              const int64_t* __restrict__ row_start, const int32_t* __restrict__ verify_len,
              const float* __restrict__ inv_temp, int V, int B, int K,
              const int32_t* __restrict__ prev_token, const int32_t* __restrict__ tokens,
              const float* __restrict__ p_tok, const float* __restrict__ ref_max,
              const float* __restrict__ ref_sum, const float* __restrict__ u_accept,
              const float2* __restrict__ tpart, int n_segs, int32_t* __restrict__ n_accepted,
              int32_t* __restrict__ out_tokens, ResInfo* __restrict__ info, unsigned* flags,
              const float* __restrict__ tok_logit = nullptr) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (b >= B) return;
  const int L = checked_len(verify_len, b, K, flags);
  const float it2 = checked_inv_temp(inv_temp, b, flags) * kLog2e;

  int n_acc = L;
  float my_tmax = 0.0f;
  double my_tz = 1.0;
  long long my_row = 0;
  for (int base_p = 0; base_p <= L; base_p += 32) {
    const int p = base_p + lane;
    bool reject = false;
    float tmax = 0.0f;
    double tz = 1.0;
    long long row = 0;
    if (p <= L) {
      row = checked_row(row_start, b, p, n_rows, flags);
      const float2* tp = tpart + (size_t)(b * (K + 1) + p) * n_segs;
      tmax = -CUDART_INF_F;
      for (int s = 0; s < n_segs; ++s) tmax = fmaxf(tmax, tp[s].x);
      tz = 0.0;
      for (int s = 0; s < n_segs; ++s) tz += (double)tp[s].y * (double)ex2((tp[s].x - tmax) * it2);
      if (!(tz > 0.0) || !isfinite(tz)) raise_flag(flags, DSPARK_FLAG_NONFINITE);
      if (p < L) {
        const int x = checked_token(tokens[(size_t)b * K + p], V, false, flags);
        // the drafted token's raw target logit: from the stored row, or
        // (LM-head verify) as the statistics pass recorded it
        const float tx = tok_logit != nullptr ? tok_logit[row] : target[(size_t)row * V + x];
        const double pt = (double)ex2((tx - tmax) * it2) / tz;
        const double pd = (double)p_tok[(size_t)b * K + p];
        // accept iff u < p_t / p_d (p_t >= p_d always accepts; p_d = 0 gives +inf)
        const double ratio = pt / pd;
        reject = !((double)u_accept[(size_t)b * K + p] < ratio);
      }
    }
    const unsigned rej = __ballot_sync(0xffffffffu, reject);
    const int first = rej ? base_p + __ffs(rej) - 1 : L;
    // the correction / bonus row is position `first` if it falls in this pass
    const int j = min(first, L);
    if (j >= base_p && j < base_p + 32) {
      my_tmax = __shfl_sync(0xffffffffu, tmax, j - base_p);
      my_tz = __shfl_sync(0xffffffffu, tz, j - base_p);
      my_row = __shfl_sync(0xffffffffu, row, j - base_p);
    }
    if (rej) {
      n_acc = first;
      break;
    }
  }
  const int j = n_acc;
  for (int p = lane; p <= K; p += 32)
    out_tokens[(size_t)b * (K + 1) + p] = (p < n_acc) ? tokens[(size_t)b * K + p] : -1;
  if (lane == 0) {
    n_accepted[b] = n_acc;
    ResInfo ri;
    ri.row = my_row;
    ri.j = j;
    ri.bonus = (j == L) ? 1 : 0;
    ri.t_max = my_tmax;
    ri.t_inv_z = (float)(1.0 / my_tz);
    ri.x_prev = -1;
    ri.d_max = 0.0f;
    ri.d_inv_z = 0.0f;
    ri.pad = 0.0f;
    if (!ri.bonus) {
      int xp = (j == 0) ? prev_token[b] : tokens[(size_t)b * K + (j - 1)];
      ri.x_prev = checked_token(xp, V, j == 0, flags);
      ri.d_max = ref_max[(size_t)b * K + j];
      const float zs = ref_sum[(size_t)b * K + j];
      if (!(zs > 0.0f) || !isfinite(zs)) raise_flag(flags, DSPARK_FLAG_NONFINITE);
      ri.d_inv_z = 1.0f / zs;
    }
    info[b] = ri;
  }
}

}  // namespace dspark
