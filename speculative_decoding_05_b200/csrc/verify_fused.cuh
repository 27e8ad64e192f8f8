// verify_fused.cuh -- the whole rejection-sampling verify of a few requests
// (B <= 4, at most 72 verified rows) in one cooperative launch, used when the
// draft's bias rows are kept so the residual needs no projection.
//
// Same arithmetic as the multi-kernel path (target_stats_kernel,
// accept_kernel, residual_bias_kernel, residual_sample_kernel), reorganised
// so that one launch replaces four and the only grid-wide waits are two
// rounds of polling on records that carry their own validity word:
//   phase 1  target-row statistics: the verified rows laid end to end are
//            cut into one contiguous range per CTA (at most V elements, so
//            it meets at most two rows); the CTA reduces its part of each row
//            to (max, sum of 2^((t - max) * log2e / T)) and stores the pairs
//            as 8-byte words {value, 1} on a line that only it writes
//            (records of several CTAs on one line, polled by every CTA, slow
//            the exchange several fold);
//   phase 2  every CTA polls, for each row, the pairs of the CTAs whose
//            ranges meet it, forms the row's (max, partition sum) and runs the
//            accept scan of every request itself, so no second exchange is
//            needed for it; CTA 0 writes n_accepted and the accepted / -1
//            entries of out_tokens;
//   phase 3  residual partials max(0, p_t - p_d) (or p_t for a bonus draw)
//            over this CTA's run of 32-row chunks; per request the CTA's
//            totals (fp64) are stored as four words {32-bit half, 1} on a
//            line of their own;
//   phase 4  the warp of request b polls every CTA's totals, finds the CTA
//            whose run holds the sample, and only that CTA resolves chunk and
//            token (two more scans over its own data) and writes the
//            correction / bonus token.
// The records are zeroed by the caller before the launch (a record is valid
// once its high word is 1).  Every wait has the 2 s limit of the library;
// running out raises DSPARK_FLAG_TIMEOUT and the kernel finishes with
// whatever it has.
#pragma once

#include "proj_tc.cuh"
#include "sample.cuh"
#include "tc_common.cuh"
#include "verify.cuh"

namespace dspark {

constexpr int kFThreads = 512;
constexpr int kFWarps = kFThreads / 32;
constexpr int kFMaxB = 4;
constexpr int kFMaxRows = 72;              // B * (K + 1)
constexpr int kFBufFloats = 24576;         // shared staging buffer (96 KB)
constexpr int kFPerLane = 5;               // CTA totals per lane: grid <= 160
constexpr int kFMaxG = 32 * kFPerLane;
constexpr int kFMaxChunks = 64;            // residual chunks of one CTA (two per lane)

struct FusedArgs {
  const float* target;
  long long n_rows;
  const int64_t* row_start;
  const int32_t* verify_len;
  const float* base;
  const float* draft_bias;
  const float* inv_temp;
  const int32_t* prev_token;
  const int32_t* tokens;
  const float* p_tok;
  const float* ref_max;
  const float* ref_sum;
  const float* u_accept;
  const float* u_res;
  int32_t* n_accepted;
  int32_t* out_tokens;
  int32_t* last_token;
  unsigned* flags;
  unsigned long long* seg_rec;  // [G][16]: row statistics of CTA c: {M_A, 1}, {S_A, 1}, {M_B, 1}, {S_B, 1}
  unsigned long long* tot_rec;  // [B][G][16]: halves of Q and P (fp64), each {half, 1}; padding
  int V, B, K, n_chunks;
};

// Words of the row-statistics records (one line per CTA), then the totals.
constexpr size_t kFSegWords = (size_t)kFMaxG * 16;
// Bytes of the records of the fused verify (zeroed before each call).
inline size_t fused_rec_bytes(int B) { return (kFSegWords + (size_t)B * kFMaxG * 16) * 8; }
inline bool fused_verify_ok(int B, int K, bool have_bias) {
  return have_bias && B >= 1 && B <= kFMaxB && B * (K + 1) <= kFMaxRows;
}

// First element of CTA c's range of the E = R V concatenated row elements.
__host__ __device__ inline long long fused_e_begin(int c, int G, long long E) {
  return E * c / G / 4 * 4;
}
// The CTA whose (non-empty) range holds element e.
__device__ inline int fused_cta_of(long long e, int G, long long E) {
  int c = (int)(e * G / E);
  if (c > G - 1) c = G - 1;
  while (c + 1 < G && fused_e_begin(c + 1, G, E) <= e) ++c;
  while (c > 0 && fused_e_begin(c, G, E) > e) --c;
  return c;
}

// Grid of the fused verify (one CTA per SM), or 0 when a CTA's run of
// chunks would not fit its scan.
// A CTA's range of the verified rows (rows V / G elements, rounded to float4)
// must stay within V elements, so that it meets at most two rows.
inline int fused_grid(int V, int rows) {
  int G = num_sms();
  if (G > kFMaxG) G = kFMaxG;
  const bool chunks_fit = (n_chunks_of(V) + G - 1) / G <= kFMaxChunks;
  const bool ranges_fit = (long long)rows * V + 4ll * G <= (long long)G * V;
  return (chunks_fit && ranges_fit) ? G : 0;
}

__device__ __forceinline__ void st_pair(unsigned long long* p, uint32_t a, uint32_t b) {
  const unsigned long long x = (1ull << 32) | a, y = (1ull << 32) | b;
  asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(x), "l"(y) : "memory");
}
__device__ __forceinline__ ulonglong2 ld_pair(const unsigned long long* p) {
  ulonglong2 v;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ bool pair_valid(ulonglong2 v) {
  return (uint32_t)(v.x >> 32) == 1u && (uint32_t)(v.y >> 32) == 1u;
}

__global__ void __launch_bounds__(kFThreads, 1) verify_fused_kernel(const FusedArgs a) {
  const bool test_skew = g_test_exchange_skew != 0;  // see common.cuh
  __shared__ int s_rofs[kFMaxB + 1];  // first flat row of request b; s_rofs[B] = rows
  __shared__ int s_len[kFMaxB];
  __shared__ float s_it2[kFMaxB];
  __shared__ int s_prev[kFMaxB];
  __shared__ long long s_rs[kFMaxB];    // row_start
  __shared__ float s_tmax[kFMaxRows];
  __shared__ double s_tz[kFMaxRows];
  __shared__ float s_tx[kFMaxRows];    // target logit of the drafted token (p < L)
  __shared__ int s_tok[kFMaxRows];     // drafted token (p < K)
  __shared__ float s_pd[kFMaxRows];    // its draft probability
  __shared__ float s_ua[kFMaxRows];    // its accept uniform
  __shared__ float s_dmax[kFMaxRows];  // draft reference max / sum of position p
  __shared__ float s_dsum[kFMaxRows];
  __shared__ ResInfo s_ri[kFMaxB];
  __shared__ float2 s_chunk[kFMaxB][kFMaxChunks];
  __shared__ float s_wm[2][kFWarps];
  __shared__ double s_ws[2][kFWarps];
  __shared__ uint64_t s_bar;             // bulk copies into s_buf
  extern __shared__ __align__(16) float s_buf[];  // kFBufFloats

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int B = a.B, K = a.K, V = a.V;

  if (tid == 0) {
    mbar_init(&s_bar, 1);
    fence_barrier_init();
  }
  uint32_t bar_phase = 0;
  // per-request inputs, one thread each (all loads in flight together)
  if (tid < B) {
    const int b = tid;
    s_len[b] = checked_len(a.verify_len, b, K, a.flags);
    s_it2[b] = checked_inv_temp(a.inv_temp, b, a.flags) * kLog2e;
    s_prev[b] = checked_token(a.prev_token[b], V, true, a.flags);
    s_rs[b] = a.row_start[b];
  }
  __syncthreads();
  if (tid == 0) {
    int r = 0;
    for (int b = 0; b < B; ++b) {
      s_rofs[b] = r;
      r += s_len[b] + 1;
    }
    s_rofs[B] = r;
  }
  __syncthreads();
  // target row of request b, position p (clamped into [0, n_rows), which
  // raises DSPARK_FLAG_BAD_LENGTH)
  auto trow_of = [&](int b, int p) {
    long long row = s_rs[b] + p;
    if (row < 0 || row >= a.n_rows) {
      raise_flag(a.flags, DSPARK_FLAG_BAD_LENGTH);
      row = row < 0 ? 0 : a.n_rows - 1;
    }
    return row;
  };
  const int R = s_rofs[B];
  auto row_of = [&](int rho, int* pb) {
    int b = 0;
    while (b + 1 < B && rho >= s_rofs[b + 1]) ++b;
    *pb = b;
    return rho - s_rofs[b];
  };

  // per-row inputs of the accept scan: loaded now, used after phase 1 (the
  // target value at the drafted token is gathered after phase 1, once the
  // token has arrived and the row is in L2)
  float g_pd = 1.0f, g_ua = 0.0f, g_dmax = 0.0f, g_dsum = 1.0f;
  int g_tokraw = 0;
  const bool g_row = tid < R;
  int g_b = 0, g_p = 0;
  if (g_row) {
    g_p = row_of(tid, &g_b);
    if (g_p < K) {
      const size_t o = (size_t)g_b * K + g_p;
      g_dmax = a.ref_max[o];
      g_dsum = a.ref_sum[o];
      if (g_p < s_len[g_b]) {
        g_tokraw = a.tokens[o];
        g_pd = a.p_tok[o];
        g_ua = a.u_accept[o];
      }
    }
  }

  // ---------------------------------------------------------------- phase 1
  // This CTA's range of the R verified rows laid end to end: float4-aligned,
  // at most V + 4 elements long (R < G), so it meets at most two rows, A and
  // B = A + 1.  One (max, sum) pair per row it meets goes out on this CTA's
  // own line.
  const long long E = (long long)R * V;
  const long long e0 = fused_e_begin(cta, G, E), e1 = fused_e_begin(cta + 1, G, E);
  {
    const int rowA = (int)min(e0 / V, (long long)max(R - 1, 0));
    const long long bnd = (long long)(rowA + 1) * V;  // first element of row B
    int bA, bB = 0;
    const int pA = row_of(rowA, &bA);
    const int pB = (rowA + 1 < R) ? row_of(rowA + 1, &bB) : 0;
    const float it2A = s_it2[bA], it2B = s_it2[bB];
    const float* tA = a.target + (size_t)trow_of(bA, pA) * V;
    const float* tB = (rowA + 1 < R) ? a.target + (size_t)trow_of(bB, pB) * V : tA;
    float mA = -CUDART_INF_F, sA = 0.0f, mB = -CUDART_INF_F, sB = 0.0f;
    // pieces of at most kFBufFloats: one or two bulk copies each (the part
    // in row A, the part in row B) into shared memory, then one pass
    for (long long p0 = e0; p0 < e1; p0 += kFBufFloats) {
      const long long p1 = min(e1, p0 + kFBufFloats);
      const long long a1 = min(p1, bnd), b0 = max(p0, bnd);
      const int nA = (int)max(0ll, a1 - p0), nB = (int)max(0ll, p1 - b0);
      if (tid == 0) {
        const uint64_t pol = policy_evict_last();  // row j is read again for the residual
        fence_proxy_async_smem();  // earlier reads of s_buf before the copies' writes
        mbar_arrive_expect_tx(&s_bar, (uint32_t)(nA + nB) * 4u);
        if (nA > 0) bulk_load(s_buf, tA + (p0 - (long long)rowA * V), (uint32_t)nA * 4u, &s_bar, pol);
        if (nB > 0) bulk_load(s_buf + nA, tB + (b0 - bnd), (uint32_t)nB * 4u, &s_bar, pol);
      }
      if (!mbar_wait(&s_bar, bar_phase)) {
        if (tid == 0) raise_flag(a.flags, DSPARK_FLAG_TIMEOUT);
      }
      bar_phase ^= 1u;
      const int n4 = (nA + nB) / 4;
      float ma = -CUDART_INF_F, mb = -CUDART_INF_F;
      for (int j = tid; j < n4; j += kFThreads) {
        const float4 x = reinterpret_cast<const float4*>(s_buf)[j];
        const float m4 = fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w));
        if (4 * j >= nA) mb = fmaxf(mb, m4);
        else ma = fmaxf(ma, m4);
      }
      float sa = 0.0f, sb = 0.0f;
      for (int j = tid; j < n4; j += kFThreads) {
        const float4 x = reinterpret_cast<const float4*>(s_buf)[j];
        const bool inB = 4 * j >= nA;
        const float m = inB ? mb : ma, it2 = inB ? it2B : it2A;
        const float e4 = ex2((x.x - m) * it2) + ex2((x.y - m) * it2) + ex2((x.z - m) * it2) +
                         ex2((x.w - m) * it2);
        if (inB) sb += e4;
        else sa += e4;
      }
      consumed(sa);  // every read of this piece has returned
      consumed(sb);
      merge_partial(mA, sA, ma, sa, it2A);
      merge_partial(mB, sB, mb, sb, it2B);
      __syncthreads();  // s_buf is refilled by the next piece
    }
    // warp, then CTA (fp64)
    const float MwA = warp_max(mA), MwB = warp_max(mB);
    const double SwA = warp_sum_d(mA == -CUDART_INF_F ? 0.0 : (double)sA * (double)ex2((mA - MwA) * it2A));
    const double SwB = warp_sum_d(mB == -CUDART_INF_F ? 0.0 : (double)sB * (double)ex2((mB - MwB) * it2B));
    if (lane == 0) {
      s_wm[0][warp] = MwA;
      s_wm[1][warp] = MwB;
      s_ws[0][warp] = SwA;
      s_ws[1][warp] = SwB;
    }
    __syncthreads();
    if (tid == 0) {
      float M[2];
      double S[2];
      for (int h = 0; h < 2; ++h) {
        const float it2 = h ? it2B : it2A;
        M[h] = -CUDART_INF_F;
        for (int w2 = 0; w2 < kFWarps; ++w2) M[h] = fmaxf(M[h], s_wm[h][w2]);
        S[h] = 0.0;
        for (int w2 = 0; w2 < kFWarps; ++w2)
          if (s_wm[h][w2] != -CUDART_INF_F) S[h] += s_ws[h][w2] * (double)ex2((s_wm[h][w2] - M[h]) * it2);
      }
      unsigned long long* r = a.seg_rec + (size_t)cta * 16;
      st_pair(r, __float_as_uint(M[0]), __float_as_uint((float)S[0]));
      st_pair(r + 2, __float_as_uint(M[1]), __float_as_uint((float)S[1]));
    }
  }
  if (g_row) {
    float tx = 0.0f;
    int tok = 0;
    if (g_p < K && g_p < s_len[g_b]) {
      tok = checked_token(g_tokraw, V, false, a.flags);
      tx = a.target[(size_t)trow_of(g_b, g_p) * V + tok];
    }
    s_tx[tid] = tx;
    s_tok[tid] = tok;
    s_pd[tid] = g_pd;
    s_ua[tid] = g_ua;
    s_dmax[tid] = g_dmax;
    s_dsum[tid] = g_dsum;
  }

  // ---------------------------------------------------------------- phase 2
  // row rho = the CTAs whose ranges meet it: [cta_of(rho V), cta_of((rho+1) V - 1)]
  for (int rho = warp; rho < R; rho += kFWarps) {
    int b;
    (void)row_of(rho, &b);
    const float it2 = s_it2[b];
    const int c_lo = fused_cta_of((long long)rho * V, G, E);
    const int c_hi = fused_cta_of((long long)(rho + 1) * V - 1, G, E);
    float2 q[kFPerLane];
    unsigned pend = 0;
#pragma unroll
    for (int i = 0; i < kFPerLane; ++i) {
      q[i] = make_float2(-CUDART_INF_F, 0.0f);
      if (c_lo + lane + 32 * i <= c_hi) pend |= 1u << i;
    }
    const uint64_t tstart = global_timer_ns();
    for (uint32_t polls = 1;; ++polls) {
      ulonglong2 m[kFPerLane];
#pragma unroll
      for (int i = 0; i < kFPerLane; ++i) {
        if (pend & (1u << i)) {
          const int c = c_lo + lane + 32 * i;
          const int slot = rho - (int)(fused_e_begin(c, G, E) / V);  // 0 or 1
          m[i] = ld_pair(a.seg_rec + (size_t)c * 16 + 2 * slot);
        }
      }
#pragma unroll
      for (int i = 0; i < kFPerLane; ++i) {
        if ((pend & (1u << i)) && pair_valid(m[i]) && !test_skew) {
          q[i] = make_float2(__uint_as_float((uint32_t)m[i].x), __uint_as_float((uint32_t)m[i].y));
          pend &= ~(1u << i);
        }
      }
      if (!__any_sync(0xffffffffu, pend != 0)) break;
      if (__any_sync(0xffffffffu, wait_expired(tstart, polls))) {
        if (lane == 0) raise_flag(a.flags, DSPARK_FLAG_TIMEOUT);
        break;
      }
    }
    float mx = -CUDART_INF_F;
#pragma unroll
    for (int i = 0; i < kFPerLane; ++i) mx = fmaxf(mx, q[i].x);
    const float tmax = warp_max(mx);
    double z = 0.0;
#pragma unroll
    for (int i = 0; i < kFPerLane; ++i)
      if (q[i].y > 0.0f) z += (double)q[i].y * (double)ex2((q[i].x - tmax) * it2);
    const double tz = warp_sum_d(z);
    if (lane == 0) {
      if (!(tz > 0.0) || !isfinite(tz)) raise_flag(a.flags, DSPARK_FLAG_NONFINITE);
      s_tmax[rho] = tmax;
      s_tz[rho] = tz;
    }
  }
  __syncthreads();

  // accept scan of request b by warp b (every CTA)
  if (warp < B) {
    const int b = warp, L = s_len[b], r0 = s_rofs[b];
    const float it2 = s_it2[b];
    int n_acc = L;
    for (int base_p = 0; base_p <= L; base_p += 32) {
      const int p = base_p + lane;
      bool reject = false;
      if (p < L) {
        const double pt = (double)ex2((s_tx[r0 + p] - s_tmax[r0 + p]) * it2) / s_tz[r0 + p];
        const double ratio = pt / (double)s_pd[r0 + p];
        reject = !((double)s_ua[r0 + p] < ratio);
      }
      const unsigned rej = __ballot_sync(0xffffffffu, reject);
      if (rej) {
        n_acc = base_p + __ffs(rej) - 1;
        break;
      }
    }
    const int j = n_acc;
    if (cta == 0) {
      for (int p = lane; p <= K; p += 32)
        if (p != j) a.out_tokens[(size_t)b * (K + 1) + p] = (p < n_acc) ? s_tok[r0 + p] : -1;
      if (lane == 0) a.n_accepted[b] = n_acc;
    }
    if (lane == 0) {
      ResInfo ri;
      ri.row = trow_of(b, j);
      ri.j = j;
      ri.bonus = (j == L) ? 1 : 0;
      ri.t_max = s_tmax[r0 + j];
      ri.t_inv_z = (float)(1.0 / s_tz[r0 + j]);
      ri.x_prev = -1;
      ri.d_max = 0.0f;
      ri.d_inv_z = 0.0f;
      ri.pad = 0.0f;
      if (!ri.bonus) {
        ri.x_prev = (j == 0) ? s_prev[b] : s_tok[r0 + j - 1];
        ri.d_max = s_dmax[r0 + j];
        const float zs = s_dsum[r0 + j];
        if (!(zs > 0.0f) || !isfinite(zs)) raise_flag(a.flags, DSPARK_FLAG_NONFINITE);
        ri.d_inv_z = 1.0f / zs;
      }
      s_ri[b] = ri;
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase 3
  const int c_begin = (int)((long long)cta * a.n_chunks / G);
  const int nch = (int)((long long)(cta + 1) * a.n_chunks / G) - c_begin;
  // the residual row's inputs of this CTA's chunk run, per request: target
  // row j, draft base and bias rows j (bulk copies into s_buf)
  const int n3 = nch * kChunk;                                  // floats per slice
  const int len3 = max(0, min(V, (c_begin + nch) * kChunk) - c_begin * kChunk);
  if (tid == 0 && len3 > 0) {
    const uint64_t pol = policy_evict_first();
    uint32_t bytes = 0;
    for (int b = 0; b < B; ++b) bytes += (s_ri[b].bonus ? 1u : 3u) * (uint32_t)len3 * 4u;
    fence_proxy_async_smem();  // phase 1's reads of s_buf before the copies' writes
    mbar_arrive_expect_tx(&s_bar, bytes);
    for (int b = 0; b < B; ++b) {
      const ResInfo& ri = s_ri[b];
      const size_t c0 = (size_t)c_begin * kChunk;
      bulk_load(s_buf + (b * 3) * n3, a.target + (size_t)ri.row * V + c0, (uint32_t)len3 * 4u, &s_bar, pol);
      if (!ri.bonus) {
        const size_t drow = ((size_t)b * K + ri.j) * (size_t)V + c0;
        bulk_load(s_buf + (b * 3 + 1) * n3, a.base + drow, (uint32_t)len3 * 4u, &s_bar, pol);
        bulk_load(s_buf + (b * 3 + 2) * n3, a.draft_bias + drow, (uint32_t)len3 * 4u, &s_bar, pol);
      }
    }
  }
  if (len3 > 0) {
    if (!mbar_wait(&s_bar, bar_phase)) {
      if (tid == 0) raise_flag(a.flags, DSPARK_FLAG_TIMEOUT);
    }
    bar_phase ^= 1u;
  }
  for (int q = warp; q < B * nch; q += kFWarps) {
    const int b = q / nch, lc = q - b * nch;
    const int vl = lc * kChunk + lane;  // element within the run
    float qv = 0.0f, pt = 0.0f;
    if (vl < len3) {
      const ResInfo& ri = s_ri[b];
      const float t = s_buf[(b * 3) * n3 + vl];
      const float bv = ri.bonus ? 0.0f : s_buf[(b * 3 + 1) * n3 + vl];
      const float bi = ri.bonus ? 0.0f : s_buf[(b * 3 + 2) * n3 + vl];
      qv = residual_q(t, bv, bi, ri, s_it2[b], &pt);
    }
    const float Q = warp_sum(qv), P = warp_sum(pt);
    if (lane == 0) s_chunk[b][lc] = make_float2(Q, P);
  }
  __syncthreads();
  if (warp < B) {
    const int b = warp;
    const int ca = 2 * lane, cb = ca + 1;
    const double q = (ca < nch ? (double)s_chunk[b][ca].x : 0.0) + (cb < nch ? (double)s_chunk[b][cb].x : 0.0);
    const double pp = (ca < nch ? (double)s_chunk[b][ca].y : 0.0) + (cb < nch ? (double)s_chunk[b][cb].y : 0.0);
    const double Qc = warp_sum_d(q), Pc = warp_sum_d(pp);
    if (lane == 0) {
      unsigned long long* r = a.tot_rec + ((size_t)b * G + cta) * 16;
      const unsigned long long qb = (unsigned long long)__double_as_longlong(Qc);
      const unsigned long long pb = (unsigned long long)__double_as_longlong(Pc);
      st_pair(r, (uint32_t)qb, (uint32_t)(qb >> 32));
      st_pair(r + 2, (uint32_t)pb, (uint32_t)(pb >> 32));
    }
  }

  // ---------------------------------------------------------------- phase 4
  if (warp < B) {
    const int b = warp;
    const ResInfo ri = s_ri[b];
    const unsigned long long* tr = a.tot_rec + (size_t)b * G * 16;
    const int per = (G + 31) / 32;
    const int c0 = min(lane * per, G), c1 = min(c0 + per, G);
    double wq[kFPerLane], wp[kFPerLane];
    unsigned pend = 0;
#pragma unroll
    for (int i = 0; i < kFPerLane; ++i) {
      wq[i] = 0.0;
      wp[i] = 0.0;
      if (c0 + i < c1) pend |= 1u << i;
    }
    const uint64_t tstart = global_timer_ns();
    for (uint32_t polls = 1;; ++polls) {
      ulonglong2 mq[kFPerLane], mp[kFPerLane];
#pragma unroll
      for (int i = 0; i < kFPerLane; ++i) {
        if (pend & (1u << i)) {
          mq[i] = ld_pair(tr + (size_t)(c0 + i) * 16);
          mp[i] = ld_pair(tr + (size_t)(c0 + i) * 16 + 2);
        }
      }
#pragma unroll
      for (int i = 0; i < kFPerLane; ++i) {
        if ((pend & (1u << i)) && pair_valid(mq[i]) && pair_valid(mp[i])) {
          wq[i] = __longlong_as_double((long long)(((mq[i].y & 0xffffffffull) << 32) | (mq[i].x & 0xffffffffull)));
          wp[i] = __longlong_as_double((long long)(((mp[i].y & 0xffffffffull) << 32) | (mp[i].x & 0xffffffffull)));
          pend &= ~(1u << i);
        }
      }
      if (!__any_sync(0xffffffffu, pend != 0)) break;
      if (__any_sync(0xffffffffu, wait_expired(tstart, polls))) {
        if (lane == 0) raise_flag(a.flags, DSPARK_FLAG_TIMEOUT);
        break;
      }
    }
    // residual mass if any, else the target distribution (bonus: Q = P)
    double lq = 0.0;
#pragma unroll
    for (int i = 0; i < kFPerLane; ++i) lq += wq[i];
    const double Qtot = warp_sum_d(lq);
    const bool use_q = Qtot > 0.0 && isfinite(Qtot);
    double lw = 0.0;
#pragma unroll
    for (int i = 0; i < kFPerLane; ++i) lw += use_q ? wq[i] : wp[i];
    const double incl = warp_incl_scan_d(lw);
    const double Z = __shfl_sync(0xffffffffu, incl, 31);
    const double T = (double)a.u_res[b] * Z;
    double start = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) start = 0.0;
    const unsigned own = __ballot_sync(0xffffffffu, start <= T && T < incl && lw > 0.0);
    int pick = -1, lastp = -1;
    double before = start, lastb = start;
    {
      double cum = start;
#pragma unroll
      for (int i = 0; i < kFPerLane; ++i) {
        const double w = use_q ? wq[i] : wp[i];
        if (pick < 0 && w > 0.0) {
          lastp = c0 + i;
          lastb = cum;
          if (cum + w > T) {
            pick = c0 + i;
            before = cum;
          }
        }
        cum += w;
      }
    }
    if (pick < 0) {
      pick = lastp;
      before = lastb;
    }
    int cstar;
    if (own) {
      const int ol = __ffs(own) - 1;
      cstar = __shfl_sync(0xffffffffu, pick, ol);
      before = __shfl_sync(0xffffffffu, before, ol);
    } else {  // no crossing (u*Z rounded to Z): the last CTA with mass
      const unsigned pos = __ballot_sync(0xffffffffu, lastp >= 0);
      const int pl = pos ? 31 - __clz(pos) : 0;
      cstar = __shfl_sync(0xffffffffu, lastp, pl);
      if (cstar < 0) cstar = 0;
      before = -CUDART_INF;
    }
    if (cstar == cta) {
      // chunk: this CTA's chunk partials, two per lane
      const int ca = 2 * lane, cb = ca + 1;
      const double wA = (ca < nch) ? (double)(use_q ? s_chunk[b][ca].x : s_chunk[b][ca].y) : 0.0;
      const double wB = (cb < nch) ? (double)(use_q ? s_chunk[b][cb].x : s_chunk[b][cb].y) : 0.0;
      const double pin = warp_incl_scan_d(wA + wB);
      double lstart = __shfl_up_sync(0xffffffffu, pin, 1);
      if (lane == 0) lstart = 0.0;
      lstart += before;
      const bool hitA = wA > 0.0 && lstart + wA > T;
      const bool hitB = wB > 0.0 && lstart + wA + wB > T;
      const unsigned h = __ballot_sync(0xffffffffu, hitA || hitB);
      int chunk;
      double before2;
      if (h) {
        const int hl = __ffs(h) - 1;
        chunk = __shfl_sync(0xffffffffu, hitA ? ca : cb, hl);
        before2 = __shfl_sync(0xffffffffu, hitA ? lstart : lstart + wA, hl);
      } else {
        const unsigned hp = __ballot_sync(0xffffffffu, wA > 0.0 || wB > 0.0);
        const int hl = hp ? 31 - __clz(hp) : 0;
        chunk = __shfl_sync(0xffffffffu, (wB > 0.0) ? cb : ca, hl);
        if (!hp) chunk = 0;
        before2 = -CUDART_INF;
      }
      // token: the chunk's 32 entries, recomputed
      const int v = (c_begin + chunk) * kChunk + lane;
      const int vl = chunk * kChunk + lane;
      const bool valid = vl < len3;
      double e = 0.0;
      if (valid) {
        const float t = s_buf[(b * 3) * n3 + vl];
        const float bv = ri.bonus ? 0.0f : s_buf[(b * 3 + 1) * n3 + vl];
        const float bi = ri.bonus ? 0.0f : s_buf[(b * 3 + 2) * n3 + vl];
        float pt;
        const float qv = residual_q(t, bv, bi, ri, s_it2[b], &pt);
        e = (double)(use_q ? qv : pt);
      }
      const int pl = pick_lane(e, before2, T);
      if (lane == pl) {
        if (!(Z > 0.0) || !isfinite(Z)) raise_flag(a.flags, DSPARK_FLAG_NONFINITE);
        const int tok = valid ? v : 0;
        a.out_tokens[(size_t)b * (K + 1) + ri.j] = tok;
        if (a.last_token != nullptr) a.last_token[b] = tok;
      }
    }
  }
}

}  // namespace dspark
