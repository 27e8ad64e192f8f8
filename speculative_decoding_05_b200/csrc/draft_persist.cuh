// draft_persist.cuh -- persistent Markov-head draft for small batches
// (B <= 16): all K sequential positions in one launch.
//
// One CTA per SM owns a contiguous range of 128-row vocabulary tiles for
// the whole call.  The first tiles of the range stay resident in shared
// memory for all K positions; the rest stream from L2 through a TMA ring
// whose producer runs ahead across positions (the tiles do not depend on
// the sampled tokens).  Per position:
//   1. gather U[x_{k-1}] for the B requests into the MMA B operand
//      (N = 16 rows, zero-padded);
//   2. tcgen05 MMAs D[v, b] = W_tile[v, :] . u_b (M = 128 vocabulary rows,
//      N = 16, K = r), one TMEM slot per tile;
//   3. epilogue (thread = vocabulary row): a = base + bias, per 32-row chunk
//      the softmax partial (max, sum exp) per request via warp shuffles,
//      the bias values to a scratch row (so the sampler needs no W), and a
//      per-CTA partial;
//   4. grid barrier (bounded spin on a counter in the workspace);
//   5. every CTA samples every request redundantly in three levels (CTA
//      partials -> chunk partials of the chosen CTA -> the 32 stored values
//      of the chosen chunk), so the next position starts without a second
//      barrier; CTA 0 writes the outputs.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer,
// warps 4..7 epilogue + sampler (TMEM lane quarters 0..3); warps 2..3 idle.
#pragma once

#include "proj_tc.cuh"
#include "sample.cuh"

namespace dspark {

constexpr int kPThreads = 256;
constexpr int kPN = 16;            // MMA N: requests, zero-padded
constexpr int kPMaxB = 16;
constexpr int kPStages = 5;        // streaming ring: 16 KB K-blocks
constexpr int kPMaxTiles = 16;     // tiles per CTA (one 16-column TMEM slot each)
constexpr int kPResidentBytes = 131072;
constexpr int kPTmemCols = 256;
constexpr int kPEpiWarp0 = 4;      // first epilogue warp
constexpr int kPEpiThreads = 128;

struct PersistArgs {
  const float* base;
  const __nv_bfloat16* U;
  const int32_t* prev_token;
  const float* inv_temp;
  const float* u_draft;
  int32_t* tokens;
  float* p_tok;
  float* lse;
  float* ref_max;
  float* ref_sum;
  float* draft_logits;
  float2* part;      // [B][n_chunks]
  float2* cta_part;  // [B][G]
  float* bias_buf;   // [B][V] scratch, used when draft_bias is NULL
  float* draft_bias; // [B][K][V] or NULL
  unsigned* flags;
  unsigned* grid_counter;
  int V, r, B, K, n_chunks, n_tiles;
};

__host__ __device__ inline int p_tile_begin(int cta, int G, int n_tiles) {
  return (int)((long long)cta * n_tiles / G);
}

inline size_t persist_smem_bytes(int r) {
  const int nkb = r / 64;
  const int tile = nkb * kStageBytes;
  const int nres = kPResidentBytes / tile;
  return 1024 + (size_t)nres * tile + (size_t)kPStages * kStageBytes + (size_t)nkb * 2048 + 1024;
}

// epilogue-group barrier (warps 4..7 only)
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kPEpiThreads) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Merge softmax partial (A, s) into (M, S) (both relative to their own max).
__device__ __forceinline__ void merge_partial(float& M, float& S, float A, float s, float it2) {
  if (A == -CUDART_INF_F) return;
  const float Mn = fmaxf(M, A);
  S = S * ex2((M - Mn) * it2) + s * ex2((A - Mn) * it2);
  M = Mn;
}

__global__ void __launch_bounds__(kPThreads, 1)
draft_persist_kernel(const __grid_constant__ CUtensorMap tm_w, const PersistArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nkb = p.r >> 6;
  const int tile_bytes = nkb * kStageBytes;
  const int max_res = kPResidentBytes / tile_bytes;
  const int G = gridDim.x, cta = blockIdx.x;
  const int t0 = p_tile_begin(cta, G, p.n_tiles), t1 = p_tile_begin(cta + 1, G, p.n_tiles);
  const int nt = t1 - t0;
  const int nres = min(nt, max_res);

  uint8_t* sRes = sm;
  uint8_t* sRing = sRes + max_res * tile_bytes;
  uint8_t* sU = sRing + kPStages * kStageBytes;
  uint64_t* ringFull = reinterpret_cast<uint64_t*>(sU + nkb * 2048);
  uint64_t* ringEmpty = ringFull + kPStages;
  uint64_t* dFull = ringEmpty + kPStages;   // [kPMaxTiles]
  uint64_t* uReady = dFull + kPMaxTiles;
  uint64_t* resReady = uReady + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(resReady + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_tok = const_cast<int*>(reinterpret_cast<volatile int*>(s_abort + 1));  // [kPMaxB]
  float* s_wm = reinterpret_cast<float*>(s_tok + kPMaxB);                        // [4][kPMaxB]
  float* s_ws = s_wm + 4 * kPMaxB;                                                // [4][kPMaxB]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = p.B, K = p.K, V = p.V;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(&ringFull[i], 1);
      mbar_init(&ringEmpty[i], 1);
    }
    for (int i = 0; i < kPMaxTiles; ++i) mbar_init(&dFull[i], 1);
    mbar_init(uReady, 1);
    mbar_init(resReady, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kPTmemCols);
  // zero the padded request rows of the B operand once (rows >= B stay zero)
  for (int i = threadIdx.x; i < nkb * 2048 / 16; i += kPThreads)
    reinterpret_cast<uint4*>(sU)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      if (nres > 0) {
        mbar_arrive_expect_tx(resReady, (uint32_t)(nres * tile_bytes));
        for (int i = 0; i < nres; ++i)
          for (int kb = 0; kb < nkb; ++kb)
            tma_load_2d_hint(sRes + i * tile_bytes + kb * kStageBytes, &tm_w, resReady, kb * 64,
                             (t0 + i) * kTileN, pol);
      }
      int it = 0;
      for (int k = 0; k < K && !*s_abort; ++k) {
        for (int i = nres; i < nt && !*s_abort; ++i) {
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % kPStages;
            const uint32_t ph = (uint32_t)(it / kPStages) & 1u;
            if (!mbar_wait(&ringEmpty[s], ph ^ 1u)) {
              *s_abort = 1;
              raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
              break;
            }
            mbar_arrive_expect_tx(&ringFull[s], kStageBytes);
            tma_load_2d_hint(sRing + s * kStageBytes, &tm_w, &ringFull[s], kb * 64,
                             (t0 + i) * kTileN, pol);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kTileN, kPN);
      const uint32_t res0 = smem_u32(sRes), ring0 = smem_u32(sRing), u0 = smem_u32(sU);
      int it = 0;
      bool ok = nres == 0 || mbar_wait(resReady, 0);
      for (int k = 0; k < K && ok; ++k) {
        if (!mbar_wait(uReady, (uint32_t)k & 1u) || *s_abort) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int i = 0; i < nt && ok; ++i) {
          const uint32_t d = tmem + (uint32_t)(i * kPN);
          for (int kb = 0; kb < nkb; ++kb) {
            uint32_t a_base;
            int s = -1;
            if (i < nres) {
              a_base = res0 + i * tile_bytes + kb * kStageBytes;
            } else {
              s = it % kPStages;
              const uint32_t ph = (uint32_t)(it / kPStages) & 1u;
              ++it;
              if (!mbar_wait(&ringFull[s], ph)) {
                ok = false;
                break;
              }
              tc_fence_after();
              a_base = ring0 + s * kStageBytes;
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(d, sdesc_sw128(a_base + kk * 32), sdesc_sw128(u0 + kb * 2048 + kk * 32),
                          idesc, (kb | kk) != 0);
            if (s >= 0) mma_commit(&ringEmpty[s]);
          }
          mma_commit(&dFull[i]);
        }
      }
      if (!ok) {
        *s_abort = 1;
        raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
      }
    }
  } else if (warp >= kPEpiWarp0) {
    // ------------------------------------------------ epilogue + sampler
    const int et = threadIdx.x - kPEpiWarp0 * 32;  // 0..127
    const int ew = warp - kPEpiWarp0;              // 0..3
    const int quarter = warp & 3;                  // TMEM lane quarter
    float it2[kPMaxB], itv[kPMaxB];
#pragma unroll
    for (int b = 0; b < kPMaxB; ++b) {
      itv[b] = (b < B) ? checked_inv_temp(p.inv_temp, b, p.flags) : 1.0f;
      it2[b] = itv[b] * kLog2e;
    }
    const int cpr = p.r >> 3;  // 16-byte chunks per U row
    for (int k = 0; k < K; ++k) {
      // 1. previous-token rows of U -> operand B (rows < B)
      for (int q = et; q < B * cpr; q += kPEpiThreads) {
        const int n = q / cpr, c = q % cpr;
        int x = (k == 0) ? p.prev_token[n] : s_tok[n];
        if (k == 0) x = checked_token(x, V, true, p.flags);
        uint4 val = make_uint4(0, 0, 0, 0);
        if (x >= 0) val = __ldg(reinterpret_cast<const uint4*>(p.U + (size_t)x * p.r) + c);
        const int kb = c >> 3, j = c & 7;
        *reinterpret_cast<uint4*>(sU + kb * 2048 + n * 128 + ((j ^ (n & 7)) << 4)) = val;
      }
      fence_proxy_async_smem();
      epi_sync();
      if (et == 0) mbar_arrive(uReady);

      // 2.-3. epilogue per tile
      float wm[kPMaxB], ws[kPMaxB];
#pragma unroll
      for (int b = 0; b < kPMaxB; ++b) {
        wm[b] = -CUDART_INF_F;
        ws[b] = 0.0f;
      }
      for (int i = 0; i < nt; ++i) {
        if (!mbar_wait(&dFull[i], (uint32_t)k & 1u)) {
          *s_abort = 1;
          raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
        }
        tc_fence_after();
        float d[16];
        tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(i * kPN), d);
        const int v = (t0 + i) * kTileN + quarter * 32 + lane;
        const bool valid = v < V;
        const int chunk = v >> 5;
#pragma unroll
        for (int b = 0; b < kPMaxB; ++b) {
          if (b >= B) break;
          const size_t row = ((size_t)b * K + k) * (size_t)V;
          const float bv = valid ? p.base[row + v] : 0.0f;
          const float a = valid ? bv + d[b] : -CUDART_INF_F;
          const float A = warp_max(a);
          const float e = valid ? ex2(((bv - A) + d[b]) * it2[b]) : 0.0f;
          const float s = warp_sum(e);
          if (valid) {
            if (p.draft_bias != nullptr) p.draft_bias[row + v] = d[b];
            else p.bias_buf[(size_t)b * V + v] = d[b];
            if (p.draft_logits != nullptr) p.draft_logits[row + v] = a * itv[b];
          }
          if (lane == 0 && chunk < p.n_chunks) {
            p.part[(size_t)b * p.n_chunks + chunk] = make_float2(A, s);
            merge_partial(wm[b], ws[b], A, s, it2[b]);
          }
        }
      }
      tc_fence_before();
      // per-CTA partial of each request
      if (lane == 0) {
#pragma unroll
        for (int b = 0; b < kPMaxB; ++b) {
          s_wm[ew * kPMaxB + b] = wm[b];
          s_ws[ew * kPMaxB + b] = ws[b];
        }
      }
      epi_sync();
      if (et < B) {
        const int b = et;
        float M = -CUDART_INF_F, S = 0.0f;
        for (int w2 = 0; w2 < 4; ++w2)
          merge_partial(M, S, s_wm[w2 * kPMaxB + b], s_ws[w2 * kPMaxB + b], it2[b]);
        p.cta_part[(size_t)b * G + cta] = make_float2(M, S);
      }
      // 4. grid barrier
      epi_sync();
      if (et == 0) {
        __threadfence();
        atomicAdd(p.grid_counter, 1u);
        const unsigned target = (unsigned)(k + 1) * (unsigned)G;
        const uint64_t tstart = global_timer_ns();
        while (ld_acquire_u32(p.grid_counter) < target) {
          if (global_timer_ns() - tstart > kWaitLimitNs) {
            *s_abort = 1;
            raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
            break;
          }
        }
        __threadfence();
      }
      epi_sync();
      if (*s_abort) {
        if (et == 0 && k + 1 < K) mbar_arrive(uReady);  // release the MMA thread
        break;
      }

      // 5. redundant three-level sampler: warp ew handles requests ew, ew+4, ...
      for (int b = ew; b < B; b += 4) {
        const double u = (double)p.u_draft[(size_t)b * K + k];
        const float2* cp = p.cta_part + (size_t)b * G;
        // level 1: CTA partials, contiguous CTA ranges per lane
        const int per = (G + 31) / 32;
        const int c0 = min(lane * per, G), c1 = min(c0 + per, G);
        float m = -CUDART_INF_F;
        for (int c = c0; c < c1; ++c) m = fmaxf(m, __ldcg(&cp[c]).x);
        const float M = warp_max(m);
        double wsum = 0.0;
        for (int c = c0; c < c1; ++c) {
          const float2 q = __ldcg(&cp[c]);
          wsum += (q.x == -CUDART_INF_F) ? 0.0 : (double)(q.y * ex2((q.x - M) * it2[b]));
        }
        const double incl = warp_incl_scan_d(wsum);
        const double Z = __shfl_sync(0xffffffffu, incl, 31);
        const double T = u * Z;
        const double excl = incl - wsum;
        // lane owning the target (intervals [excl, incl) of consecutive lanes)
        const double prev_incl = __shfl_up_sync(0xffffffffu, incl, 1);
        const double start = lane == 0 ? 0.0 : prev_incl;
        unsigned own = __ballot_sync(0xffffffffu, start <= T && T < incl && wsum > 0.0);
        int cstar = -1;
        double before = 0.0;
        if (own) {
          const int ol = __ffs(own) - 1;
          if (lane == ol) {
            double cum = start;
            int lastp = -1;
            double lastb = start;
            for (int c = c0; c < c1; ++c) {
              const float2 q = __ldcg(&cp[c]);
              const double w = (q.x == -CUDART_INF_F) ? 0.0 : (double)(q.y * ex2((q.x - M) * it2[b]));
              if (w > 0.0) {
                lastp = c;
                lastb = cum;
              }
              if (cum + w > T && w > 0.0) {
                cstar = c;
                before = cum;
                break;
              }
              cum += w;
            }
            if (cstar < 0) {
              cstar = lastp;
              before = lastb;
            }
          }
          cstar = __shfl_sync(0xffffffffu, cstar, ol);
          before = __shfl_sync(0xffffffffu, before, ol);
        }
        bool fallback = false;
        if (cstar < 0) {  // no crossing (u*Z rounded to Z): last CTA with mass
          const unsigned pos = __ballot_sync(0xffffffffu, wsum > 0.0);
          const int pl = pos ? 31 - __clz(pos) : 0;
          int lastc = -1;
          if (lane == pl)
            for (int c = c0; c < c1; ++c)
              if (__ldcg(&cp[c]).x != -CUDART_INF_F && __ldcg(&cp[c]).y > 0.0f) lastc = c;
          cstar = __shfl_sync(0xffffffffu, lastc, pl);
          if (cstar < 0) cstar = 0;
          fallback = true;
        }
        (void)excl;
        // level 2: chunk partials of CTA cstar (<= 64 chunks, two per lane)
        const int ch0 = p_tile_begin(cstar, G, p.n_tiles) * (kTileN / kChunk);
        const int ch1 = min(p_tile_begin(cstar + 1, G, p.n_tiles) * (kTileN / kChunk), p.n_chunks);
        const float2* pp = p.part + (size_t)b * p.n_chunks;
        double wA = 0.0, wB = 0.0;
        const int ca = ch0 + 2 * lane, cb2 = ca + 1;
        if (ca < ch1) {
          const float2 q = __ldcg(&pp[ca]);
          wA = (q.x == -CUDART_INF_F) ? 0.0 : (double)(q.y * ex2((q.x - M) * it2[b]));
        }
        if (cb2 < ch1) {
          const float2 q = __ldcg(&pp[cb2]);
          wB = (q.x == -CUDART_INF_F) ? 0.0 : (double)(q.y * ex2((q.x - M) * it2[b]));
        }
        const double pin = warp_incl_scan_d(wA + wB);
        const double lstart = before + (pin - (wA + wB));
        int chunk = -1;
        double before2 = 0.0;
        if (!fallback) {
          const bool hitA = wA > 0.0 && lstart + wA > T;
          const bool hitB = wB > 0.0 && lstart + wA + wB > T;
          const unsigned h = __ballot_sync(0xffffffffu, hitA || hitB);
          if (h) {
            const int hl = __ffs(h) - 1;
            const int myc = hitA ? ca : cb2;
            const double myb = hitA ? lstart : lstart + wA;
            chunk = __shfl_sync(0xffffffffu, myc, hl);
            before2 = __shfl_sync(0xffffffffu, myb, hl);
          }
        }
        if (chunk < 0) {  // last chunk of the CTA with positive weight
          const unsigned h = __ballot_sync(0xffffffffu, wA > 0.0 || wB > 0.0);
          const int hl = h ? 31 - __clz(h) : 0;
          const int myc = (wB > 0.0) ? cb2 : ca;
          chunk = __shfl_sync(0xffffffffu, myc, hl);
          before2 = -CUDART_INF;
          if (!h) chunk = ch0;
        }
        // level 3: the 32 stored values of the chunk
        const int v = chunk * kChunk + lane;
        const bool valid = v < V;
        double e = 0.0;
        float ef = 0.0f;
        if (valid) {
          const float bias = p.draft_bias != nullptr
                                 ? __ldcg(&p.draft_bias[((size_t)b * K + k) * (size_t)V + v])
                                 : __ldcg(&p.bias_buf[(size_t)b * V + v]);
          const float bv = p.base[((size_t)b * K + k) * (size_t)V + v];
          ef = ex2(((bv - M) + bias) * it2[b]);
          e = (double)ef;
        }
        const int pick = pick_lane(e, before2, T);
        if (lane == pick) {
          s_tok[b] = valid ? v : 0;
          if (cta == 0) {
            const size_t o = (size_t)b * K + k;
            if (!(Z > 0.0) || !isfinite(Z)) {
              raise_flag(p.flags, DSPARK_FLAG_NONFINITE);
              p.tokens[o] = 0;
              p.p_tok[o] = 0.0f;
              p.lse[o] = CUDART_NAN_F;
              p.ref_max[o] = M;
              p.ref_sum[o] = 1.0f;
            } else {
              p.tokens[o] = valid ? v : 0;
              p.p_tok[o] = (float)((double)ef / Z);
              p.lse[o] = (float)((double)M * (double)itv[b] + log(Z));
              p.ref_max[o] = M;
              p.ref_sum[o] = (float)Z;
            }
          }
        }
      }
      epi_sync();  // s_tok visible to the next position's gather
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kPTmemCols);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

inline int persist_grid(int V) {
  const int n_tiles = (V + kTileN - 1) / kTileN;
  int G = num_sms();
  if (G > n_tiles) G = n_tiles;
  return G;
}

inline bool persist_supported(int V, int r, int B) {
  if (B < 1 || B > kPMaxB || r % 64 != 0 || r < 64 || r > 256 || V % 4 != 0 || V < kTileN)
    return false;
  const int n_tiles = (V + kTileN - 1) / kTileN;
  const int G = persist_grid(V);
  return (n_tiles + G - 1) / G <= kPMaxTiles;
}

// Workspace bytes the persistent draft needs beyond the chunk partials:
// per-CTA partials and the bias rows.
inline size_t persist_extra_bytes(int V, int B) {
  return align256((size_t)B * 1024 * sizeof(float2)) + align256((size_t)B * V * sizeof(float));
}

inline dspark_status persist_launch(const CUtensorMap& tm_w, const PersistArgs& a, cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(draft_persist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)persist_smem_bytes(256));
    attr = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(persist_grid(a.V));
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = persist_smem_bytes(a.r);
  cfg.stream = s;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, draft_persist_kernel, tm_w, a) == cudaSuccess ? DSPARK_OK
                                                                                 : DSPARK_ERR_CUDA;
}

}  // namespace dspark
