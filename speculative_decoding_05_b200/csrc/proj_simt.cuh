// proj_simt.cuh -- CUDA-core (SIMT) projection kernels for small batches.
//
// One warp owns kChunk = 32 consecutive vocabulary rows (one row per lane).
// Each lane streams its W row once (16-byte vector loads, fp32 FMA
// accumulation in ascending index order: the same order as dot_row) and
// forms the bias for up to NB requests at once, then the warp reduces
// the chunk to a softmax partial with shuffles.  This is the
// "vectorised warp-shuffle GEMV" regime: B is too small for the tensor
// cores to pay, so the kernel is bound by streaming W.
#pragma once

#include "common.cuh"

namespace dspark {

// Per-request description of the verify row that gets the correction /
// bonus draw (written by the accept kernel).
struct ResInfo {
  long long row;   // target row of position j
  int j;           // 0-based position of the correction / bonus token
  int bonus;       // 1: every verified token was accepted -> draw from p_t
  int x_prev;      // token before position j (-1: none) for the draft row
  float t_max;     // target row reference max (raw logits)
  float t_inv_z;   // 1 / sum_v exp((t_v - t_max) * inv_temp)
  float d_max;     // draft row reference max (un-tempered logits)
  float d_inv_z;   // 1 / draft partition sum relative to d_max
  float pad;
};

// Residual weight max(0, p_t - p_d) of one vocabulary entry, and p_t.
__device__ __forceinline__ float residual_q(float t, float bv, float bias, const ResInfo& ri,
                                            float it2, float* pt_out) {
  float pt = ex2((t - ri.t_max) * it2) * ri.t_inv_z;
  *pt_out = pt;
  if (ri.bonus) return pt;
  float pd = ex2(((bv - ri.d_max) + bias) * it2) * ri.d_inv_z;
  return fmaxf(pt - pd, 0.0f);
}

// Gather the previous-token rows of U for NB requests into shared memory
// (fp32; zero rows for "no previous token").
template <typename TW, int NB>
__device__ __forceinline__ void gather_u_rows(const TW* __restrict__ U, const int* x, int r,
                                              float* __restrict__ u_s) {
  for (int b = 0; b < NB; ++b) {
    const int xb = x[b];
    for (int i = threadIdx.x; i < r; i += blockDim.x)
      u_s[b * r + i] = (xb >= 0) ? to_f32(U[(size_t)xb * r + i]) : 0.0f;
  }
}

// acc[b] = U[x_b] . W[v] for NB requests, same accumulation order as dot_row.
template <typename TW, int NB>
__device__ __forceinline__ void dot_rows(const TW* __restrict__ wrow, const float* __restrict__ u_s,
                                         int r, float (&acc)[NB]) {
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = 0.0f;
#pragma unroll 2
  for (int i = 0; i < r; i += 8) {
    float w8[8];
    load8(wrow + i, w8);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float4 ua = *reinterpret_cast<const float4*>(u_s + b * r + i);
      float4 ub = *reinterpret_cast<const float4*>(u_s + b * r + i + 4);
      float a = acc[b];
      a = fmaf(w8[0], ua.x, a); a = fmaf(w8[1], ua.y, a);
      a = fmaf(w8[2], ua.z, a); a = fmaf(w8[3], ua.w, a);
      a = fmaf(w8[4], ub.x, a); a = fmaf(w8[5], ub.y, a);
      a = fmaf(w8[6], ub.z, a); a = fmaf(w8[7], ub.w, a);
      acc[b] = a;
    }
  }
}

// Draft projection for position k (0-based) of requests
// [blockIdx.y*NB, +NB): per 32-row chunk c and request b the partial
// (A_c, s_c) with A_c = max_v (base + bias) and
// s_c = sum_v exp(((base_v - A_c) + bias_v) * inv_temp).
// Subtracting A_c from the base before adding the bias keeps the exponent
// of the tokens that matter exact to a few ulp of a small number.
template <typename TW, int NB>
__global__ void __launch_bounds__(256)
draft_proj_simt_kernel(const float* __restrict__ base, const TW* __restrict__ U,
                       const TW* __restrict__ W, int V, int r, int B, int K, int k,
                       const int32_t* __restrict__ prev_token, const int32_t* __restrict__ tokens,
                       const float* __restrict__ inv_temp, float* __restrict__ draft_logits,
                       float* __restrict__ draft_bias, float2* __restrict__ part, int n_chunks,
                       unsigned* flags) {
  extern __shared__ __align__(16) float u_s[];  // [NB][r]
  __shared__ int x[NB];
  __shared__ float it2[NB], it[NB];
  const int b0 = blockIdx.y * NB;
  if (threadIdx.x < NB) {
    const int b = threadIdx.x, gb = b0 + b;
    int xb = -1;
    float itb = 1.0f;
    if (gb < B) {
      xb = (k == 0) ? prev_token[gb] : tokens[(size_t)gb * K + (k - 1)];
      xb = checked_token(xb, V, /*allow_none=*/k == 0, flags);
      itb = checked_inv_temp(inv_temp, gb, flags);
    }
    x[b] = xb;
    it[b] = itb;
    it2[b] = itb * kLog2e;
  }
  __syncthreads();
  gather_u_rows<TW, NB>(U, x, r, u_s);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps_per_cta = blockDim.x >> 5;
  for (int c = blockIdx.x * warps_per_cta + warp; c < n_chunks; c += gridDim.x * warps_per_cta) {
    const int v = c * kChunk + lane;
    const bool valid = v < V;
    float acc[NB];
    if (valid) {
      dot_rows<TW, NB>(W + (size_t)v * r, u_s, r, acc);
    } else {
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = 0.0f;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int gb = b0 + b;
      if (gb >= B) break;
      const size_t row = ((size_t)gb * K + k) * (size_t)V;
      const float bv = valid ? base[row + v] : 0.0f;
      const float a = valid ? bv + acc[b] : -CUDART_INF_F;
      const float A = warp_max(a);
      const float e = valid ? ex2(((bv - A) + acc[b]) * it2[b]) : 0.0f;
      const float s = warp_sum(e);
      if (lane == 0) part[(size_t)gb * n_chunks + c] = make_float2(A, s);
      if (draft_logits != nullptr && valid) draft_logits[row + v] = a * it[b];
      if (draft_bias != nullptr && valid) draft_bias[row + v] = acc[b];
    }
  }
}

// Residual projection: for each request its correction row j (from the
// accept kernel), per 32-row chunk the sums (sum_v q_v, sum_v p_t(v)) with
// q = max(0, p_t - p_d) (q = p_t for a bonus draw).
template <typename TW, int NB>
__global__ void __launch_bounds__(256)
residual_proj_simt_kernel(const float* __restrict__ target, const float* __restrict__ base,
                          const TW* __restrict__ U, const TW* __restrict__ W, int V, int r, int B,
                          int K, const ResInfo* __restrict__ info,
                          const float* __restrict__ inv_temp, float2* __restrict__ rpart,
                          int n_chunks, unsigned* flags) {
  extern __shared__ __align__(16) float u_s[];  // [NB][r]
  __shared__ int x[NB];
  __shared__ float it2[NB];
  __shared__ ResInfo ri[NB];
  const int b0 = blockIdx.y * NB;
  if (threadIdx.x < NB) {
    const int b = threadIdx.x, gb = b0 + b;
    if (gb < B) {
      ri[b] = info[gb];
      it2[b] = checked_inv_temp(inv_temp, gb, flags) * kLog2e;
      x[b] = ri[b].bonus ? -1 : ri[b].x_prev;
    } else {
      x[b] = -1;
      it2[b] = kLog2e;
    }
  }
  __syncthreads();
  gather_u_rows<TW, NB>(U, x, r, u_s);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps_per_cta = blockDim.x >> 5;
  for (int c = blockIdx.x * warps_per_cta + warp; c < n_chunks; c += gridDim.x * warps_per_cta) {
    const int v = c * kChunk + lane;
    const bool valid = v < V;
    float acc[NB];
    if (valid) {
      dot_rows<TW, NB>(W + (size_t)v * r, u_s, r, acc);
    } else {
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = 0.0f;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int gb = b0 + b;
      if (gb >= B) break;
      float q = 0.0f, pt = 0.0f;
      if (valid) {
        const float t = target[(size_t)ri[b].row * V + v];
        const float bv = ri[b].bonus ? 0.0f : base[((size_t)gb * K + ri[b].j) * (size_t)V + v];
        q = residual_q(t, bv, acc[b], ri[b], it2[b], &pt);
      }
      const float Q = warp_sum(q), P = warp_sum(pt);
      if (lane == 0) rpart[(size_t)gb * n_chunks + c] = make_float2(Q, P);
    }
  }
}

// Residual partials when the draft's bias rows are available: the draft row
// at position j is rebuilt from base + bias without touching W.  Grid
// (chunk groups, B); one warp per 32-row chunk, lane = vocabulary row.
__global__ void __launch_bounds__(256)
residual_bias_kernel(const float* __restrict__ target, const float* __restrict__ base,
                     const float* __restrict__ draft_bias, int V, int K,
                     const ResInfo* __restrict__ info, const float* __restrict__ inv_temp,
                     float2* __restrict__ rpart, int n_chunks, unsigned* flags) {
  const int b = blockIdx.y;
  const ResInfo ri = info[b];
  const float it2 = checked_inv_temp(inv_temp, b, flags) * kLog2e;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* trow = target + (size_t)ri.row * V;
  const size_t drow = ((size_t)b * K + (ri.bonus ? 0 : ri.j)) * (size_t)V;
  for (int c = blockIdx.x * 8 + warp; c < n_chunks; c += gridDim.x * 8) {
    const int v = c * kChunk + lane;
    float q = 0.0f, pt = 0.0f;
    if (v < V) {
      const float t = trow[v];
      const float bv = ri.bonus ? 0.0f : base[drow + v];
      const float bias = ri.bonus ? 0.0f : draft_bias[drow + v];
      q = residual_q(t, bv, bias, ri, it2, &pt);
    }
    const float Q = warp_sum(q), P = warp_sum(pt);
    if (lane == 0) rpart[(size_t)b * n_chunks + c] = make_float2(Q, P);
  }
}

}  // namespace dspark
