// draft_persist.cuh -- persistent Markov-head draft for small batches
// (B <= 16): all K sequential positions in one launch.
//
// One CTA per SM owns a contiguous range of 128-row vocabulary tiles for
// the whole call.  Its W tiles stream from L2 through one deep TMA ring
// whose producer runs ahead across positions: the tiles do not depend on
// the sampled tokens, so while the grid waits at a barrier and samples,
// the ring already fills with the next position's tiles (as good as
// keeping that much of W resident).  The base-logit rows of the CTA's
// range are bulk-copied into shared memory one position ahead by another
// producer warp.  Per position:
//   1. tcgen05 MMAs D[v, b] = W_tile[v, :] . U[x_b] (M = 128 vocabulary
//      rows, N = 16 requests zero-padded, K = r) into an 8-slot TMEM
//      accumulator ring.  The first three tiles of every CTA's range stay
//      resident in TMEM for the whole call and feed the MMA as its A operand
//      straight from tensor memory (28 MB of W on chip across the GPU), so
//      the part that streams each position (about 49 MB at V = 151936,
//      r = 256) stays L2-resident; the rest comes from the TMA ring;
//   2. epilogue (thread = vocabulary row): a = base + bias, per 32-row chunk
//      the softmax partial (max, sum exp) per request via warp shuffles,
//      the bias values to a scratch row (so the sampler needs no W), and a
//      per-CTA partial;
//   3. grid barrier: a release reduction on one counter, relaxed polling
//      with a time limit, one acquire fence;
//   4. every CTA samples every request redundantly in three dependent
//      loads (CTA partials -> chunk partials of the chosen CTA -> the 32
//      stored values of the chosen chunk), so the next position needs no
//      second barrier; the sampling warp writes U[x_k] straight into the
//      MMA operand; CTA 0 writes the outputs.
//
// Warp roles: warp 0 W producer (TMA), warp 1 TMEM allocator + MMA issuer,
// warp 2 base producer (bulk copies), warps 4..7 epilogue + sampler (TMEM
// lane quarters 0..3); warp 3 idle.
#pragma once

#include "proj_tc.cuh"
#include "sample.cuh"

namespace dspark {

constexpr int kPThreads = 256;
constexpr int kPN = 16;          // MMA N: requests, zero-padded
constexpr int kPMaxB = 16;
constexpr int kPMaxTiles = 16;   // tiles per CTA
constexpr int kPTmemCols = 512;
constexpr int kPDSlots = 8;      // accumulator ring: 8 x 16 TMEM columns
constexpr int kPACol = 128;      // first TMEM column of the resident W tiles
constexpr int kPMaxTmemTiles = 3;  // W tiles resident in TMEM (128 columns each)
constexpr int kPGroup = 1;       // tiles whose MMAs are issued together
constexpr int kPEpiWarp0 = 4;    // first epilogue warp
constexpr int kPEpiThreads = 128;
constexpr int kPMaxG = 256;      // grid limit of the sampler's register arrays
constexpr int kPMinStages = 4;
constexpr int kPMaxStages = 24;
constexpr int kPSmemLimit = 232448;  // 227 KB of dynamic shared memory

struct PersistArgs {
  const float* base;
  const __nv_bfloat16* U;
  const __nv_bfloat16* W;
  const int32_t* prev_token;
  const float* inv_temp;
  const float* u_draft;
  int32_t* tokens;
  float* p_tok;
  float* lse;
  float* ref_max;
  float* ref_sum;
  float* draft_logits;
  float2* part;       // [B][n_chunks]
  float2* cta_part;   // [B][G]
  float* bias_buf;    // [B][V] scratch, used when draft_bias is NULL
  float* draft_bias;  // [B][K][V] or NULL
  unsigned* flags;
  unsigned* grid_counter;
  int V, r, B, K, n_chunks, n_tiles;
  int max_nt;         // tiles of the largest CTA range
  int n_stages;       // W ring stages (16 KB each)
};

__host__ __device__ inline int p_tile_begin(int cta, int G, int n_tiles) {
  return (int)((long long)cta * n_tiles / G);
}

struct PersistLayout {
  int G, max_nt, n_stages;
  size_t u_bytes, base_bytes, smem;
};

inline int persist_grid(int V) {
  const int n_tiles = (V + kTileN - 1) / kTileN;
  int G = num_sms();
  if (G > n_tiles) G = n_tiles;
  if (G > kPMaxG) G = kPMaxG;
  return G;
}

// Up to this many requests (at r = 256) the persistent draft runs its
// projection as a CUDA-core GEMV; above it, on tcgen05 with N = 16.
constexpr int kSimtMaxB = 2;
inline bool gemv_path(int r, int B) { return B <= kSimtMaxB && r == 256; }

// Work split of the GEMV variant: 32-row chunks, a contiguous run per CTA.
constexpr int kGRank = 256;
constexpr int kGTailBytes = kChunk * kGRank * 2;    // 16 KB: the tail chunk's W rows
constexpr int kGMaxChunks = 64;                     // chunks of one CTA (two per lane in level 2)
constexpr int kGPerLane = 5;                        // CTA partials per lane in level 1
constexpr int kGMaxG = 32 * kGPerLane;              // grid limit of the GEMV variant
// Each CTA's partial record sits on its own 128-byte line: with 148 pollers
// reading every record, records that share lines slow the exchange several
// fold (the writes queue behind the reads of the shared line).
constexpr int kGRecWords = 16;                      // 8-byte words per record line
// W chunks (32 rows, 16 KB) kept in shared memory for the whole call, beside
// the 16 in TMEM; the rest of a CTA's chunks stream through the ring.
constexpr int kGResChunks = 8;
constexpr int kGMaxUnits = 12;                      // units per warp and position

// First chunk of CTA c: runs balanced to within one chunk.
__host__ __device__ inline int gemv_chunk_begin(int cta, int G, int n_chunks) {
  return (int)((long long)cta * n_chunks / G);
}
// 1 when a run of nc chunks hands its last chunk to the tail warp.
__host__ __device__ inline int gemv_tail(int nc) { return (nc % 4 == 1) ? 1 : 0; }

// Largest chunk run of a CTA, and the most 128-row tiles its GEMV warps take.
inline void gemv_runs(int n_chunks, int G, int* max_chunks, int* max_tiles) {
  const int q = n_chunks / G, rem = n_chunks % G;
  *max_chunks = q + (rem ? 1 : 0);
  int mt = 0;
  for (int nc = q; nc <= *max_chunks; ++nc) {
    const int tiles = (nc - gemv_tail(nc) + 3) / 4;
    if (tiles > mt) mt = tiles;
  }
  *max_tiles = mt;
}

inline PersistLayout persist_layout(int V, int r, int B) {
  PersistLayout L;
  const int n_tiles = (V + kTileN - 1) / kTileN;
  L.G = persist_grid(V);
  L.max_nt = (n_tiles + L.G - 1) / L.G;
  if (gemv_path(r, B)) {
    const int n_chunks = n_chunks_of(V);
    int G = num_sms();
    if (G > n_chunks) G = n_chunks;
    if (G > kGMaxG) G = kGMaxG;
    int max_chunks;
    L.G = G;
    gemv_runs(n_chunks, G, &max_chunks, &L.max_nt);
    // tail rows, sBias [B][rows_cap] + sBase [2][B][rows_cap] + sPart [B][part_cap]
    const size_t rows_cap = (size_t)L.max_nt * kTileN + kChunk, part_cap = (size_t)L.max_nt * 4 + 1;
    L.u_bytes = kGTailBytes + (size_t)kGResChunks * kStageBytes;
    L.base_bytes = (size_t)3 * B * rows_cap * 4 + (size_t)B * part_cap * 8 + 16 +
                   (size_t)2 * B * kGMaxChunks * 8;  // + chunk weights and prefix sums (fp64)
  } else {
    L.u_bytes = (size_t)(r / 64) * 2048;
    L.base_bytes = (((size_t)B * L.max_nt * kTileN * 4) + 1023) & ~size_t(1023);
  }
  const size_t fixed = 1024 /*align*/ + L.u_bytes + L.base_bytes + 2048 /*barriers, scratch*/;
  L.n_stages = fixed >= (size_t)kPSmemLimit ? 0 : (int)((kPSmemLimit - fixed) / kStageBytes);
  if (L.n_stages > kPMaxStages) L.n_stages = kPMaxStages;
  L.smem = fixed + (size_t)L.n_stages * kStageBytes;
  return L;
}

// epilogue-group barrier (warps 4..7 only)
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kPEpiThreads) : "memory");
}


// Write U[x] (or zeros) into row n of the 128-byte swizzled K-major B
// operand, one 16-byte chunk per lane step.
__device__ __forceinline__ void store_u_row(uint8_t* sU, const __nv_bfloat16* U, int x, int n, int r,
                                            int lane) {
  const int cpr = r >> 3;
  for (int c = lane; c < cpr; c += 32) {
    uint4 val = make_uint4(0, 0, 0, 0);
    if (x >= 0) val = __ldg(reinterpret_cast<const uint4*>(U + (size_t)x * r) + c);
    const int kb = c >> 3, j = c & 7;
    *reinterpret_cast<uint4*>(sU + kb * 2048 + n * 128 + ((j ^ (n & 7)) << 4)) = val;
  }
}

// Grid barrier of position k, called by one thread per CTA: a release
// reduction on the counter, relaxed polling with a time limit, then one
// acquire fence.  Returns false on timeout (DSPARK_FLAG_TIMEOUT raised).
__device__ __forceinline__ bool persist_grid_barrier(unsigned* counter, int k, int G,
                                                     unsigned* flags) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(counter) : "memory");
  const unsigned target = (unsigned)(k + 1) * (unsigned)G;
  const uint64_t tstart = global_timer_ns();
  bool ok = true;
  for (uint32_t polls = 1;; ++polls) {
    unsigned seen;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(counter) : "memory");
    if (seen >= target) break;
    if (wait_expired(tstart, polls)) {
      raise_flag(flags, DSPARK_FLAG_TIMEOUT);
      ok = false;
      break;
    }
  }
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
  return ok;
}

// Redundant three-level sampler of request b at position k, one full warp:
// CTA partials -> chunk partials of the chosen CTA -> the 32 stored bias
// values of the chosen chunk.  Every CTA computes the same token; CTA 0
// writes the outputs.  Returns the token (in every lane).
__device__ __noinline__ int persist_sample(const PersistArgs& p, int b, int k, int G, int cta,
                                           float it2b, float itvb) {
  const int lane = threadIdx.x & 31;
  const int K = p.K, V = p.V;
        const double u = (double)p.u_draft[(size_t)b * K + k];
        const float2* cp = p.cta_part + (size_t)b * G;
        // level 1: CTA partials (contiguous ranges of at most 8 CTAs per lane)
        const int per = (G + 31) / 32;
        const int c0 = min(lane * per, G), c1 = min(c0 + per, G);
        float2 q[kPMaxG / 32];
#pragma unroll
        for (int i = 0; i < kPMaxG / 32; ++i)
          q[i] = (c0 + i < c1) ? __ldcg(&cp[c0 + i]) : make_float2(-CUDART_INF_F, 0.0f);
        float m = -CUDART_INF_F;
#pragma unroll
        for (int i = 0; i < kPMaxG / 32; ++i) m = fmaxf(m, q[i].x);
        const float M = warp_max(m);
        double wsum = 0.0;
#pragma unroll
        for (int i = 0; i < kPMaxG / 32; ++i) wsum += partial_weight(q[i], M, it2b);
        const double incl = warp_incl_scan_d(wsum);
        const double Z = __shfl_sync(0xffffffffu, incl, 31);
        const double T = u * Z;
        double start = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) start = 0.0;
        const unsigned own = __ballot_sync(0xffffffffu, start <= T && T < incl && wsum > 0.0);
        int cstar = -1;
        double before = 0.0;
        {
          double cum = start, lastb = start, pb = start;
          int pick = -1, lastp = -1;
#pragma unroll
          for (int i = 0; i < kPMaxG / 32; ++i) {
            const double w = partial_weight(q[i], M, it2b);
            if (pick < 0 && w > 0.0) {
              lastp = c0 + i;
              lastb = cum;
              if (cum + w > T) {
                pick = c0 + i;
                pb = cum;
              }
            }
            cum += w;
          }
          if (pick < 0) {
            pick = lastp;
            pb = lastb;
          }
          if (own) {
            const int ol = __ffs(own) - 1;
            cstar = __shfl_sync(0xffffffffu, pick, ol);
            before = __shfl_sync(0xffffffffu, pb, ol);
          } else {  // no crossing (u*Z rounded to Z): last CTA with mass
            const unsigned pos = __ballot_sync(0xffffffffu, lastp >= 0);
            const int pl = pos ? 31 - __clz(pos) : 0;
            cstar = __shfl_sync(0xffffffffu, lastp, pl);
            before = -CUDART_INF;
            if (cstar < 0) cstar = 0;
          }
        }
        // level 2: chunk partials of CTA cstar (<= 64 chunks, two per lane)
        const int ch0 = p_tile_begin(cstar, G, p.n_tiles) * (kTileN / kChunk);
        const int ch1 = min(p_tile_begin(cstar + 1, G, p.n_tiles) * (kTileN / kChunk), p.n_chunks);
        const float2* pp = p.part + (size_t)b * p.n_chunks;
        const int ca = ch0 + 2 * lane, cb2 = ca + 1;
        const float2 qa = (ca < ch1) ? __ldcg(&pp[ca]) : make_float2(-CUDART_INF_F, 0.0f);
        const float2 qb = (cb2 < ch1) ? __ldcg(&pp[cb2]) : make_float2(-CUDART_INF_F, 0.0f);
        const double wA = partial_weight(qa, M, it2b), wB = partial_weight(qb, M, it2b);
        const double pin = warp_incl_scan_d(wA + wB);
        double lstart = __shfl_up_sync(0xffffffffu, pin, 1);
        if (lane == 0) lstart = 0.0;
        lstart += before;
        int chunk = -1;
        double before2 = 0.0;
        {
          const bool hitA = wA > 0.0 && lstart + wA > T;
          const bool hitB = wB > 0.0 && lstart + wA + wB > T;
          const unsigned h = __ballot_sync(0xffffffffu, hitA || hitB);
          if (h) {
            const int hl = __ffs(h) - 1;
            const int myc = hitA ? ca : cb2;
            const double myb = hitA ? lstart : lstart + wA;
            chunk = __shfl_sync(0xffffffffu, myc, hl);
            before2 = __shfl_sync(0xffffffffu, myb, hl);
          } else {  // rounding: last chunk of the CTA with positive weight
            const unsigned hp = __ballot_sync(0xffffffffu, wA > 0.0 || wB > 0.0);
            const int hl = hp ? 31 - __clz(hp) : 0;
            const int myc = (wB > 0.0) ? cb2 : ca;
            chunk = __shfl_sync(0xffffffffu, myc, hl);
            if (!hp) chunk = ch0;
            before2 = -CUDART_INF;
          }
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
          ef = ex2(((bv - M) + bias) * it2b);
          e = (double)ef;
        }
        const int pick = pick_lane(e, before2, T);
        const int x = __shfl_sync(0xffffffffu, valid ? v : 0, pick);
        if (lane == pick && cta == 0) {
          const size_t o = (size_t)b * K + k;
          if (!(Z > 0.0) || !isfinite(Z)) {
            raise_flag(p.flags, DSPARK_FLAG_NONFINITE);
            p.tokens[o] = 0;
            p.p_tok[o] = 0.0f;
            p.lse[o] = CUDART_NAN_F;
            p.ref_max[o] = M;
            p.ref_sum[o] = 1.0f;
          } else {
            p.tokens[o] = x;
            p.p_tok[o] = (float)((double)ef / Z);
            p.lse[o] = (float)((double)M * (double)itvb + log(Z));
            p.ref_max[o] = M;
            p.ref_sum[o] = (float)Z;
          }
        }
  return x;
}

__global__ void __launch_bounds__(kPThreads, 1)
draft_persist_kernel(const __grid_constant__ CUtensorMap tm_w, const PersistArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nkb = p.r >> 6;
  const int G = gridDim.x, cta = blockIdx.x;
  const int t0 = p_tile_begin(cta, G, p.n_tiles), t1 = p_tile_begin(cta + 1, G, p.n_tiles);
  const int nt = t1 - t0;
  const int B = p.B, K = p.K, V = p.V;
  const int S = p.n_stages;
  const int base_stride = p.max_nt * kTileN;  // floats per request in sBase
  const int nres = min(nt, kPMaxTmemTiles);   // tiles resident in TMEM

  uint8_t* sRing = sm;
  uint8_t* sU = sRing + S * kStageBytes;
  float* sBase = reinterpret_cast<float*>(sU + nkb * 2048);
  uint8_t* misc = reinterpret_cast<uint8_t*>(sBase) +
                  ((((size_t)B * base_stride * 4) + 1023) & ~size_t(1023));
  uint64_t* ringFull = reinterpret_cast<uint64_t*>(misc);
  uint64_t* ringEmpty = ringFull + kPMaxStages;
  uint64_t* dFull = ringEmpty + kPMaxStages;  // [kPDSlots]
  uint64_t* dEmpty = dFull + kPDSlots;        // [kPDSlots]
  uint64_t* uReady = dEmpty + kPDSlots;
  uint64_t* baseFull = uReady + 1;
  uint64_t* baseEmpty = baseFull + 1;
  uint64_t* mmaDrain = baseEmpty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mmaDrain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_wm = reinterpret_cast<float*>(tmem_slot + 2);  // [4][kPMaxB]
  float* s_ws = s_wm + 4 * kPMaxB;                        // [4][kPMaxB]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&ringFull[i], 1);
      mbar_init(&ringEmpty[i], 1);
    }
    for (int i = 0; i < kPDSlots; ++i) {
      mbar_init(&dFull[i], 1);
      mbar_init(&dEmpty[i], 4);
    }
    mbar_init(uReady, 1);
    mbar_init(baseFull, 1);
    mbar_init(baseEmpty, 1);
    mbar_init(mmaDrain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kPTmemCols);
  // operand B of position 1: U[prev_token] rows, zero rows past B
  for (int i = threadIdx.x; i < nkb * 2048 / 16; i += kPThreads)
    reinterpret_cast<uint4*>(sU)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (warp >= kPEpiWarp0) {
    const int ew = warp - kPEpiWarp0;
    for (int b = ew; b < B; b += 4) {
      const int x = checked_token(p.prev_token[b], V, true, p.flags);
      store_u_row(sU, p.U, x, b, p.r, lane);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp >= kPEpiWarp0) {
    // resident W tiles -> TMEM: lane = tile row, 32-bit column c holds the
    // bf16 pair (2c, 2c+1) of the row (the A-operand layout of a
    // tensor-memory MMA)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    for (int i = 0; i < nres; ++i) {
      const int v = (t0 + i) * kTileN + row;
      const uint4* src = reinterpret_cast<const uint4*>(p.W + (size_t)(v < V ? v : 0) * p.r);
      for (int g = 0; g < (p.r >> 6); ++g) {
        uint32_t regs[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 val = (v < V) ? __ldg(src + g * 8 + q) : make_uint4(0, 0, 0, 0);
          regs[4 * q] = val.x;
          regs[4 * q + 1] = val.y;
          regs[4 * q + 2] = val.z;
          regs[4 * q + 3] = val.w;
        }
        tmem_st32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(kPACol + i * 128 + g * 32),
                  regs);
      }
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ------------------------------------------------ W producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int it = 0;
      for (int k = 0; k < K && !*s_abort; ++k) {
        for (int g0 = nres; g0 < nt && !*s_abort; g0 += kPGroup) {
          const int gn = min(kPGroup, nt - g0);
          for (int kb = 0; kb < nkb && !*s_abort; ++kb) {
            for (int j = 0; j < gn; ++j, ++it) {
              const int s = it % S;
              const uint32_t ph = (uint32_t)(it / S) & 1u;
              if (!mbar_wait(&ringEmpty[s], ph ^ 1u)) {
                *s_abort = 1;
                raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
                break;
              }
              mbar_arrive_expect_tx(&ringFull[s], kStageBytes);
              tma_load_2d_hint(sRing + s * kStageBytes, &tm_w, &ringFull[s], kb * 64,
                               (t0 + g0 + j) * kTileN, pol);
            }
          }
        }
      }
      // tail: the MMAs' release of the last stages is an asynchronous arrive
      // on this CTA's barriers; wait for it before the CTA may exit (after
      // an abort: for the copies still in flight)
      if (!*s_abort) wait_ring_released(ringEmpty, S, it, p.flags);
      else drain_ring_loads(ringFull, S, it);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kTileN, kPN);
      const uint32_t ring0 = smem_u32(sRing), u0 = smem_u32(sU);
      int it = 0;
      bool ok = true;
      for (int k = 0; k < K && ok; ++k) {
        if (!mbar_wait_spin(uReady, (uint32_t)k & 1u) || *s_abort) {
          ok = false;
          break;
        }
        tc_fence_after();
        // groups: the TMEM-resident tiles, then streamed tiles kPGroup at a time
        for (int g0 = 0; g0 < nt && ok;) {
          const bool resident = g0 < nres;
          const int gn = min(kPGroup, (resident ? nres : nt) - g0);
          uint32_t dcol[kPGroup];
          for (int j = 0; j < gn && ok; ++j) {
            const int i = g0 + j, slot = i % kPDSlots;
            const int per_step = (nt - slot + kPDSlots - 1) / kPDSlots;  // uses per position
            const uint32_t use = (uint32_t)(k * per_step + i / kPDSlots);
            ok = mbar_wait_spin(&dEmpty[slot], (use & 1u) ^ 1u);
            dcol[j] = tmem + (uint32_t)(slot * kPN);
          }
          if (!ok) break;
          tc_fence_after();
          if (resident) {
            for (int kb = 0; kb < nkb; ++kb) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = sdesc_sw128(u0 + kb * 2048 + kk * 32);
                for (int j = 0; j < gn; ++j)
                  mma_bf16_ts(dcol[j], tmem + (uint32_t)(kPACol + (g0 + j) * 128 + (kb * 4 + kk) * 8),
                              bd, idesc, (kb | kk) != 0);
              }
            }
          } else {
            for (int kb = 0; kb < nkb && ok; ++kb) {
              int st[kPGroup];
              for (int j = 0; j < gn; ++j, ++it) {
                st[j] = it % S;
                if (!mbar_wait_spin(&ringFull[st[j]], (uint32_t)(it / S) & 1u)) {
                  ok = false;
                  break;
                }
              }
              if (!ok) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = sdesc_sw128(u0 + kb * 2048 + kk * 32);
                for (int j = 0; j < gn; ++j)
                  mma_bf16_ss(dcol[j], sdesc_sw128(ring0 + st[j] * kStageBytes + kk * 32), bd, idesc,
                              (kb | kk) != 0);
              }
              for (int j = 0; j < gn; ++j) mma_commit(&ringEmpty[st[j]]);
            }
          }
          if (!ok) break;
          for (int j = 0; j < gn; ++j) mma_commit(&dFull[(g0 + j) % kPDSlots]);
          g0 += gn;
        }
      }
      if (!ok) {
        *s_abort = 1;
        raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
      }
      drain_mma(mmaDrain);
    }
  } else if (warp == 2) {
    // ------------------------------------------------ base producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int v0 = t0 * kTileN;
      const int nval = min(nt * kTileN, V - v0);
      const uint32_t bytes = (uint32_t)nval * 4u;
      int last = -1;  // last position whose rows were requested
      for (int k = 0; k < K && !*s_abort; ++k) {
        if (!mbar_wait(baseEmpty, ((uint32_t)k & 1u) ^ 1u)) {
          *s_abort = 1;
          raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(baseFull, bytes * (uint32_t)B);
        for (int b = 0; b < B; ++b)
          bulk_load(sBase + (size_t)b * base_stride, p.base + ((size_t)b * K + k) * (size_t)V + v0,
                    bytes, baseFull, pol);
        last = k;
      }
      // after an abort the last rows may still be landing
      if (*s_abort && last >= 0) mbar_wait(baseFull, (uint32_t)last & 1u);
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
    if (et == 0) mbar_arrive(uReady);  // operand B of position 1 is in place
    for (int k = 0; k < K; ++k) {
      // ---- epilogue over the CTA's tiles
      float wm[kPMaxB], ws[kPMaxB];
#pragma unroll
      for (int b = 0; b < kPMaxB; ++b) {
        wm[b] = -CUDART_INF_F;
        ws[b] = 0.0f;
      }
      bool ok = mbar_wait_spin(baseFull, (uint32_t)k & 1u);
      for (int i = 0; i < nt; ++i) {
        const int slot = i % kPDSlots;
        const int per_step = (nt - slot + kPDSlots - 1) / kPDSlots;
        const uint32_t use = (uint32_t)(k * per_step + i / kPDSlots);
        ok = ok && mbar_wait_spin(&dFull[slot], use & 1u);
        if (!ok) {
          *s_abort = 1;
          raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
        }
        tc_fence_after();
        float d[16];
        tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(slot * kPN), d);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dEmpty[slot]);
        const int vl = i * kTileN + quarter * 32 + lane;  // row within the CTA range
        const int v = t0 * kTileN + vl;
        const bool valid = v < V;
        const int chunk = v >> 5;
#pragma unroll
        for (int b = 0; b < kPMaxB; ++b) {
          if (b >= B) break;
          const size_t row = ((size_t)b * K + k) * (size_t)V;
          const float bv = valid ? sBase[(size_t)b * base_stride + vl] : 0.0f;
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
      if (lane == 0) {
#pragma unroll
        for (int b = 0; b < kPMaxB; ++b) {
          s_wm[ew * kPMaxB + b] = wm[b];
          s_ws[ew * kPMaxB + b] = ws[b];
        }
      }
      epi_sync();
      if (et == 0) mbar_arrive(baseEmpty);  // sBase may take the next position
      if (et < B) {
        const int b = et;
        float M = -CUDART_INF_F, Sm = 0.0f;
        for (int w2 = 0; w2 < 4; ++w2)
          merge_partial(M, Sm, s_wm[w2 * kPMaxB + b], s_ws[w2 * kPMaxB + b], it2[b]);
        p.cta_part[(size_t)b * G + cta] = make_float2(M, Sm);
      }
      // ---- grid barrier
      epi_sync();
      if (et == 0 && !persist_grid_barrier(p.grid_counter, k, G, p.flags)) *s_abort = 1;
      epi_sync();
      if (*s_abort) {
        if (et == 0 && k + 1 < K) mbar_arrive(uReady);  // release the MMA thread
        break;
      }

      // ---- redundant sampler: warp ew handles requests ew, ew+4, ...
      for (int b = ew; b < B; b += 4) {
        const int x = persist_sample(p, b, k, G, cta, it2[b], itv[b]);
        // operand B of the next position: U[x] into row b
        if (k + 1 < K) store_u_row(sU, p.U, x, b, p.r, lane);
      }
      fence_proxy_async_smem();
      epi_sync();
      if (et == 0 && k + 1 < K) mbar_arrive(uReady);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kPTmemCols);
}

// ---------------------------------------------------------------------------
// GEMV variant for one or two requests (r = 256)
// ---------------------------------------------------------------------------
//
// An N = 16 tcgen05 MMA costs about as much as a much wider one, so for one
// or two requests the projection is a GEMV on the CUDA cores.  It is laid
// out "transposed": lane l of a warp owns the K slice [8l, 8l+8) of every
// row, so the previous-token vector U[x] stays in eight registers per
// request, each lane accumulates the dot products of 32 rows at once, and
// a 31-shuffle butterfly hands lane l the finished bias of row l.
//
// Work split: the vocabulary is cut into 32-row chunks and every CTA owns
// a contiguous run of them, balanced to within one chunk.  Eight GEMV warps
// take the CTA's chunks four at a time as 128-row tiles (warp (h, q) takes
// rows 32q..32q+31 of the tiles of parity h).  When a run has one chunk
// more than a multiple of four, that last chunk goes to warp 2, which keeps
// its W rows in shared memory for the whole call, instead of giving one GEMV
// warp a fifth tile.  Memory plan of the GEMV warps: four W tiles per SM
// resident in TMEM for the whole call, stored in the same transposed order
// (lane = K slice, four 32-bit columns = 8 bf16 per row) and read back with
// tcgen05.ld; the rest streams through the TMA ring; base rows are
// bulk-copied one position ahead (double-buffered).
//
// One round of global exchange per position, without fences or counters:
// after its tiles each CTA stores its softmax partial as two 8-byte words
// {value, position + 1}.  The warp of request b polls the G partials of b
// until every word carries the current position (relaxed loads, re-reading
// only the stale ones), finds the CTA whose range
// holds the sample, and only that CTA resolves the chunk and the token from
// its own shared memory (chunk partials, bias and base values of its rows).
// It writes the outputs, starts pulling U[x] into L2, and publishes
// {position + 1, token} as one 8-byte word; one thread per CTA polls that
// word and every warp then loads its slice of U[x] for the next position.
// The partials are double-buffered by position parity: a CTA publishes
// position k+2 only after every CTA has read position k's partials (a token
// of k+1 needs every CTA's partial of k+1, which each CTA stores after it has
// read k's).
//
// Warp roles: warp 0 TMEM allocator + W producer (TMA), warp 1 base
// producer (bulk copies), warp 2 tail chunk, warps 3..10 GEMV (TMEM lane
// quarter = warp % 4; warps 3..6 take the even tiles, 7..10 the odd ones).
constexpr int kGThreads = 352;
constexpr int kGTailWarp = 2;
constexpr int kGCompWarp0 = 3;
constexpr int kGSyncThreads = 288;  // warps 2..10
constexpr int kGMaxB = 2;
constexpr int kGMaxTmemTiles = 4;
constexpr int kGSlots = 9;                          // per-warp partials: 8 GEMV warps + tail warp

__device__ __forceinline__ void gemv_sync() {
  asm volatile("bar.sync 1, %0;" ::"r"(kGSyncThreads) : "memory");
}
// the same barrier, returning whether any participating thread passed true
__device__ __forceinline__ bool gemv_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(kGSyncThreads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void st_rec(unsigned long long* p, uint32_t lo, uint32_t seq) {
  const unsigned long long v = ((unsigned long long)seq << 32) | lo;
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_rec(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
// the pair of 8-byte words at p (16-byte aligned); each word is read as one
// single-copy-atomic access, the pair as two
__device__ __forceinline__ ulonglong2 ld_rec2(const unsigned long long* p) {
  ulonglong2 v;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2::evict_last [%0];" ::"l"(p));
}

// lane l receives sum over lanes of v[l] (butterfly transpose-reduce)
__device__ __forceinline__ float transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

// c + w * u for the low / high bf16 of two packed pairs, accumulated in
// fp32: the product of two bf16 values is exact in fp32, so this equals
// fmaf(float(w), float(u), c) with no conversion instructions.
__device__ __forceinline__ float fma_bf16_lo(uint32_t w, uint32_t u, float c) {
  float d;
  asm("{\n\t.reg .b16 wl, wh, ul, uh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\tmov.b32 {ul, uh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, wl, ul, %3;\n\t}"
      : "=f"(d) : "r"(w), "r"(u), "f"(c));
  return d;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t w, uint32_t u, float c) {
  float d;
  asm("{\n\t.reg .b16 wl, wh, ul, uh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\tmov.b32 {ul, uh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, wh, uh, %3;\n\t}"
      : "=f"(d) : "r"(w), "r"(u), "f"(c));
  return d;
}

// pr[b][row] += sum_{e<8} w_e * u_e over the 8 bf16 packed in q and in u[b]
// (ascending e, one rounding per step), for all NB requests (the kernel runs
// with exactly NB requests: no runtime test splits the unrolled FMA stream)
template <int NB>
__device__ __forceinline__ void gemv8(uint4 q, const uint32_t (&u)[NB][4], float (&pr)[NB][32], int row) {
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    float a = pr[b][row];
    a = fma_bf16_lo(q.x, u[b][0], a); a = fma_bf16_hi(q.x, u[b][0], a);
    a = fma_bf16_lo(q.y, u[b][1], a); a = fma_bf16_hi(q.y, u[b][1], a);
    a = fma_bf16_lo(q.z, u[b][2], a); a = fma_bf16_hi(q.z, u[b][2], a);
    a = fma_bf16_lo(q.w, u[b][3], a); a = fma_bf16_hi(q.w, u[b][3], a);
    pr[b][row] = a;
  }
}

// u[b] = the 8 bf16 of U[x_b][8 lane .. 8 lane + 7], packed (zeros for x < 0)
template <int NB>
__device__ __forceinline__ void load_u_slice(const __nv_bfloat16* U, const int (&x)[NB], int B, int lane,
                                             uint32_t (&u)[NB][4]) {
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    uint4 val = make_uint4(0, 0, 0, 0);
    if (b < B && x[b] >= 0) val = __ldg(reinterpret_cast<const uint4*>(U + (size_t)x[b] * kGRank) + lane);
    u[b][0] = val.x;
    u[b][1] = val.y;
    u[b][2] = val.z;
    u[b][3] = val.w;
  }
}

struct GemvRecs {
  unsigned long long* cta;  // [2][B][G][16]: {M, seq}, {S, seq}, then padding to 128 B
  unsigned long long* tok;  // [B][16]: {position + 1, token}, then padding
};

__device__ __forceinline__ void backoff_spin_u64(const unsigned long long* p, uint32_t seq,
                                                 unsigned long long* out, bool* timed_out) {
  const uint64_t tstart = global_timer_ns();
  for (uint32_t polls = 1;; ++polls) {
    const unsigned long long v = ld_rec(p);
    if ((uint32_t)(v >> 32) == seq) {
      *out = v;
      return;
    }
    if (wait_expired(tstart, polls)) {
      *timed_out = true;
      *out = 0;
      return;
    }
  }
}


template <int NB>
__global__ void __launch_bounds__(kGThreads, 1)
draft_gemv_kernel(const __grid_constant__ CUtensorMap tm_w, const PersistArgs p, const GemvRecs rec) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t test_skew = (uint32_t)g_test_exchange_skew;
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = gridDim.x, cta = blockIdx.x;
  constexpr int B = NB;  // launched with exactly NB requests
  const int K = p.K, V = p.V;
  const int S = p.n_stages;
  const int c_begin = gemv_chunk_begin(cta, G, p.n_chunks);
  const int nc = gemv_chunk_begin(cta + 1, G, p.n_chunks) - c_begin;  // chunks of this CTA
  const int tail = gemv_tail(nc);
  const int mainc = nc - tail;                   // chunks of the GEMV warps
  const int nt = (mainc + 3) / 4;                // their 128-row tiles
  const int v0 = c_begin * kChunk;               // first vocabulary row of this CTA
  const int nrows = min(nc * kChunk, V - v0);    // valid rows of this CTA
  const int main_rows = min(mainc * kChunk, nrows);
  const int rows_cap = p.max_nt * kTileN + kChunk;  // row slots per request in sBias / sBase
  const int part_cap = p.max_nt * 4 + 1;            // chunk slots per request in sPart
  const int nres = min(nt, kGMaxTmemTiles);
  const int n_tm = min(4 * nres, mainc);             // chunks held in TMEM (tiles 0..nres-1)
  const int n_res = min(kGResChunks, mainc - n_tm);  // chunks held in shared memory
  const int n_str = mainc - n_tm - n_res;            // chunks streamed every position

  uint8_t* sRing = sm;
  uint8_t* sTail = sRing + S * kStageBytes;                                  // [32 rows][512 B]
  uint8_t* sRes = sTail + kGTailBytes;                                       // [kGResChunks][16 KB]
  float* sBias = reinterpret_cast<float*>(sRes + kGResChunks * kStageBytes); // [B][rows_cap]
  float* sBase = sBias + (size_t)B * rows_cap;                               // [2][B][rows_cap]
  float2* sPart = reinterpret_cast<float2*>(sBase + (size_t)2 * B * rows_cap);  // [B][part_cap]
  // after sPart: the chunk weights and prefix sums (2 B kGMaxChunks doubles,
  // one float2 slot each), then the barriers and small arrays
  uint8_t* misc = reinterpret_cast<uint8_t*>(sPart + (size_t)B * part_cap + (size_t)2 * B * kGMaxChunks);
  misc = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(misc) + 15) & ~uintptr_t(15));
  uint64_t* ringFull = reinterpret_cast<uint64_t*>(misc);
  uint64_t* ringEmpty = ringFull + kPMaxStages;
  uint64_t* baseFull = ringEmpty + kPMaxStages;  // [2]
  uint64_t* baseEmpty = baseFull + 2;            // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(baseEmpty + 2);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_wm = reinterpret_cast<float*>(tmem_slot + 2);  // [kGSlots][kGMaxB]
  float* s_ws = s_wm + kGSlots * kGMaxB;                  // [kGSlots][kGMaxB]
  volatile int* s_i = reinterpret_cast<volatile int*>(s_ws + kGSlots * kGMaxB);  // [4]
  float* s_ud = const_cast<float*>(reinterpret_cast<volatile float*>(s_i + 4));   // [B][K] draft uniforms
  int* s_units = reinterpret_cast<int*>(s_ud + kGMaxB * 64);  // [9][kGMaxUnits] (type, index, chunk)
  int* s_nunits = s_units + 9 * kGMaxUnits;                    // [9]
  float* s_acta = reinterpret_cast<float*>(s_nunits + 12);     // [kGMaxB] CTA max per request
  // fill number of each ring stage (consecutive fills of a stage go to
  // different warps; see tag_wait)
  volatile int* s_tag = reinterpret_cast<volatile int*>(s_acta + kGMaxB);  // [kPMaxStages]
  // chunk weights relative to the CTA max and their inclusive prefix sums
  double* s_cw = reinterpret_cast<double*>(sPart + (size_t)B * part_cap);  // [B][kGMaxChunks]
  double* s_cp = s_cw + (size_t)B * kGMaxChunks;                                     // [B][kGMaxChunks]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&ringFull[i], 1);
      mbar_init(&ringEmpty[i], 1);  // one consumer warp per fill
    }
    for (int i = 0; i < kPMaxStages; ++i) s_tag[i] = -1;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&baseFull[i], 1);
      mbar_init(&baseEmpty[i], 1);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kPTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ W producer (streamed tiles)
    if (lane == 0 && n_str > 0) {
      // Stage = one streamed chunk, 32 whole W rows (16 KB, contiguous in
      // global memory): one bulk copy, consumed by one warp.  (A swizzled 2D
      // box of 128 rows x 128 B per stage arrived several times slower.)
      // Rows past V are not read.
      const uint64_t pol = policy_evict_last();
      int it = 0;
      for (int k = 0; k < K && !*s_abort; ++k) {
        for (int sc = 0; sc < n_str && !*s_abort; ++sc, ++it) {
          const int s = it % S;
          if (!mbar_wait(&ringEmpty[s], ((uint32_t)(it / S) & 1u) ^ 1u)) {
            *s_abort = 1;
            raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
            break;
          }
          s_tag[s] = it;
          const int row0 = v0 + (n_tm + n_res + sc) * kChunk;
          const int nr = max(0, min(kChunk, V - row0));
          if (nr > 0) {
            mbar_arrive_expect_tx(&ringFull[s], (uint32_t)nr * (kGRank * 2));
            bulk_load(sRing + s * kStageBytes, p.W + (size_t)row0 * kGRank, (uint32_t)nr * (kGRank * 2),
                      &ringFull[s], pol);
          } else {
            mbar_arrive(&ringFull[s]);
          }
        }
      }
      drain_ring_loads(ringFull, S, it);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ base producer (double-buffered)
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t bytes = (uint32_t)nrows * 4u;
      int issued = 0;
      for (int k = 0; k < K && !*s_abort; ++k) {
        const int buf = k & 1;
        if (!mbar_wait(&baseEmpty[buf], ((uint32_t)(k >> 1) & 1u) ^ 1u)) {
          *s_abort = 1;
          raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&baseFull[buf], bytes * (uint32_t)B);
        for (int b = 0; b < B; ++b)
          bulk_load(sBase + ((size_t)buf * B + b) * rows_cap,
                    p.base + ((size_t)b * K + k) * (size_t)V + v0, bytes, &baseFull[buf], pol);
        ++issued;
      }
      drain_ring_loads(baseFull, 2, issued);
    }
  } else if (warp >= kGTailWarp) {
    // ------------------------------------------------ GEMV, epilogue, sampling
    const bool gemv = warp >= kGCompWarp0;
    const int cw = warp - kGCompWarp0;          // 0..7 for the GEMV warps, -1 for the tail warp
    const int slot = gemv ? cw : kGSlots - 1;   // this warp's partial slot
    const int half = cw >> 1 >> 1;              // tile parity owned by a GEMV warp
    const int quarter = warp & 3;               // TMEM lane quarter = rows 32q..32q+31 of a tile
    float it2[NB], itv[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      itv[b] = (b < B) ? checked_inv_temp(p.inv_temp, b, p.flags) : 1.0f;
      it2[b] = itv[b] * kLog2e;
    }
    if (gemv) {
      // resident tiles -> TMEM in transposed order
      for (int i = half; i < nres; i += 2) {
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t regs[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int row = v0 + i * kTileN + quarter * 32 + cb * 8 + j;
            const uint4 val = (row < V) ? __ldg(reinterpret_cast<const uint4*>(p.W + (size_t)row * kGRank) + lane)
                                        : make_uint4(0, 0, 0, 0);
            regs[4 * j] = val.x;
            regs[4 * j + 1] = val.y;
            regs[4 * j + 2] = val.z;
            regs[4 * j + 3] = val.w;
          }
          tmem_st32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(i * 128 + cb * 32), regs);
        }
      }
      tmem_st_wait();
      // this warp's shared-memory-resident chunks, row-major (512 B per row)
      for (int j = cw; j < n_res; j += 8) {
        for (int rr = 0; rr < kChunk; ++rr) {
          const int row = v0 + (n_tm + j) * kChunk + rr;
          const uint4 val = (row < V) ? __ldg(reinterpret_cast<const uint4*>(p.W + (size_t)row * kGRank) + lane)
                                      : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(sRes + j * kStageBytes + rr * (kGRank * 2) + lane * 16) = val;
        }
      }
    } else if (tail) {
      // the tail chunk's W rows -> shared memory, row-major (512 B per row)
      for (int rr = 0; rr < kChunk; ++rr) {
        const int row = v0 + main_rows + rr;
        const uint4 val = (main_rows + rr < nrows)
                              ? __ldg(reinterpret_cast<const uint4*>(p.W + (size_t)row * kGRank) + lane)
                              : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sTail + rr * (kGRank * 2) + lane * 16) = val;
      }
    }
    // Units of 32 rows (one chunk each), per warp: its TMEM chunks (rows
    // 32q..32q+31 of the tiles of parity h), its shared-memory chunks and its
    // streamed chunks (chunk j of those outside TMEM goes to warp j % 8).
    // Half 0 takes its streamed chunks first (they were fetched during the
    // previous exchange; releasing them early lets the rest of this
    // position's stream land in time), half 1 last.  Each warp takes its
    // streamed chunks in increasing order, which keeps the ring free of
    // deadlock.  Entry: (type << 24) | (index << 12) | chunk, type 0 = TMEM
    // tile, 1 = resident chunk, 2 = stream index, 3 = the tail chunk.
    if (threadIdx.x == kGTailWarp * 32) {
      for (int w = 0; w < 8; ++w) {
        const int h = w >> 2, q = (w + kGCompWarp0) & 3;
        int a_[kGMaxUnits], na = 0, r_[kGMaxUnits], nr_ = 0, st[kGMaxUnits], nst = 0;
        for (int i = h; i < nres; i += 2)
          if (4 * i + q < mainc && na < kGMaxUnits) a_[na++] = (i << 12) | (4 * i + q);
        for (int j = w; j < n_res; j += 8)
          if (nr_ < kGMaxUnits) r_[nr_++] = (1 << 24) | (j << 12) | (n_tm + j);
        for (int j = n_res; j < mainc - n_tm; ++j)
          if (j % 8 == w && nst < kGMaxUnits) st[nst++] = (2 << 24) | ((j - n_res) << 12) | (n_tm + j);
        int* ul = s_units + w * kGMaxUnits;
        int n = 0;
        if (h == 0)
          for (int t = 0; t < nst && n < kGMaxUnits; ++t) ul[n++] = st[t];
        for (int t = 0; t < max(na, nr_); ++t) {
          if (t < na && n < kGMaxUnits) ul[n++] = a_[t];
          if (t < nr_ && n < kGMaxUnits) ul[n++] = r_[t];
        }
        if (h == 1)
          for (int t = 0; t < nst && n < kGMaxUnits; ++t) ul[n++] = st[t];
        s_nunits[w] = n;
      }
      s_units[8 * kGMaxUnits] = (3 << 24) | mainc;
      s_nunits[8] = tail;
    }
    // the draft uniforms of every position, staged so the sampling step
    // never waits on a global load
    for (int i = threadIdx.x - kGTailWarp * 32; i < B * K; i += kGSyncThreads) s_ud[i] = p.u_draft[i];
    // U[prev_token] slice of this lane
    uint32_t u[NB][4];
    {
      int x[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) x[b] = (b < B) ? checked_token(p.prev_token[b], V, true, p.flags) : -1;
      load_u_slice<NB>(p.U, x, B, lane, u);
    }
    tc_fence_before();
    gemv_sync();
    tc_fence_after();

    for (int k = 0; k < K; ++k) {
      const int buf = k & 1, par = k & 1;
      const uint32_t seq = (uint32_t)k + 1u;
      const float* bse = sBase + (size_t)buf * B * rows_cap;
      float wm[NB], ws[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        wm[b] = -CUDART_INF_F;
        ws[b] = 0.0f;
      }
      bool ok = mbar_wait_spin(&baseFull[buf], (uint32_t)(k >> 1) & 1u);

      const int* ul = s_units + (gemv ? cw : 8) * kGMaxUnits;
      const int n_units = s_nunits[gemv ? cw : 8];
      for (int n = 0; n < n_units; ++n) {
        const int e = ul[n];
        const int type = e >> 24, idx = (e >> 12) & 0xfff, c = e & 0xfff;
        float pr[NB][32];
#pragma unroll
        for (int b = 0; b < NB; ++b)
#pragma unroll
          for (int j = 0; j < 32; ++j) pr[b][j] = 0.0f;
        if (type == 0) {
          // eight 16-column groups (4 rows each), the next group's
          // tcgen05.ld in flight while the current one is multiplied
          const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(idx * 128);
          uint32_t wa[16], wb[16];
          tmem_ld16_issue(ta, wa);
          tmem_ld16_wait(wa);
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            uint32_t (&cur)[16] = (g & 1) ? wb : wa;
            uint32_t (&nxt)[16] = (g & 1) ? wa : wb;
            if (g + 1 < 8) tmem_ld16_issue(ta + (uint32_t)((g + 1) * 16), nxt);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              gemv8<NB>(make_uint4(cur[4 * j], cur[4 * j + 1], cur[4 * j + 2], cur[4 * j + 3]), u, pr, g * 4 + j);
            if (g + 1 < 8) tmem_ld16_wait(nxt);
          }
        } else {
          // 32 rows of 512 B in shared memory: a resident chunk, a ring
          // stage or the tail chunk
          int it = 0;
          const uint8_t* buf;
          if (type == 2) {
            it = k * n_str + idx;
            ok = ok && tag_wait(s_tag + it % S, it) &&
                 mbar_wait_spin(&ringFull[it % S], (uint32_t)(it / S) & 1u);
            buf = sRing + (it % S) * kStageBytes;
          } else {
            buf = (type == 1) ? sRes + idx * kStageBytes : sTail;
          }
          // four groups of 8 rows: the barriers keep the compiler from
          // hoisting all 32 shared loads (128 registers) at once
#pragma unroll
          for (int rr = 0; rr < 32; ++rr) {
            if ((rr & 7) == 0 && rr > 0) asm volatile("" ::: "memory");
            const uint4 q = *reinterpret_cast<const uint4*>(buf + rr * (kGRank * 2) + lane * 16);
            gemv8<NB>(q, u, pr, rr);
          }
          if (type == 2) {
            // release the stage once every lane's reads of it have returned
#pragma unroll
            for (int b = 0; b < NB; ++b)
#pragma unroll
              for (int j = 0; j < 32; ++j) consumed(pr[b][j]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&ringEmpty[it % S]);
          }
        }
        // this lane's row: its bias (butterfly), kept in shared memory and,
        // when asked for, in global memory
        const int vl = c * kChunk + lane;
        const bool valid = vl < nrows;
        const int v = v0 + vl;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float bias = transpose_reduce32(pr[b], lane);
          sBias[(size_t)b * rows_cap + vl] = bias;
          if (valid) {
            const size_t row = ((size_t)b * K + k) * (size_t)V;
            if (p.draft_bias != nullptr) p.draft_bias[row + v] = bias;
            if (p.draft_logits != nullptr)
              p.draft_logits[row + v] = (bse[(size_t)b * rows_cap + vl] + bias) * itv[b];
          }
        }
      }
      // softmax partial of every unit (chunk), four units at a time so that
      // their shuffle chains overlap
      __syncwarp();
      for (int n0 = 0; n0 < n_units; n0 += 4) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float bv[4], bi[4], am[4], es[4];
          bool ok4[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int n = n0 + j;
            const int vl = ((n < n_units) ? (ul[n] & 0xfff) : 0) * kChunk + lane;
            ok4[j] = n < n_units && vl < nrows;
            bv[j] = ok4[j] ? bse[(size_t)b * rows_cap + vl] : 0.0f;
            bi[j] = ok4[j] ? sBias[(size_t)b * rows_cap + vl] : 0.0f;
            am[j] = ok4[j] ? bv[j] + bi[j] : -CUDART_INF_F;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int j = 0; j < 4; ++j) am[j] = fmaxf(am[j], __shfl_xor_sync(0xffffffffu, am[j], o));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            es[j] = ok4[j] ? ex2(((bv[j] - am[j]) + bi[j]) * it2[b]) : 0.0f;
            // from here on the slot holds the row's weight relative to its
            // chunk's max (the sampling step's last level reads it)
            if (n0 + j < n_units) sBias[(size_t)b * rows_cap + ((ul[n0 + j] & 0xfff) * kChunk + lane)] = es[j];
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int j = 0; j < 4; ++j) es[j] += __shfl_xor_sync(0xffffffffu, es[j], o);
          if (lane == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int n = n0 + j;
              if (n >= n_units) break;
              sPart[(size_t)b * part_cap + (ul[n] & 0xfff)] = make_float2(am[j], es[j]);
              merge_partial(wm[b], ws[b], am[j], es[j], it2[b]);
            }
          }
        }
      }
      if (!ok) {
        *s_abort = 1;
        raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
      }
      if (lane == 0) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          s_wm[slot * kGMaxB + b] = wm[b];
          s_ws[slot * kGMaxB + b] = ws[b];
        }
      }
      gemv_sync();
      // publish this CTA's partial of every request
      if (cw == 0 && lane < B) {
        const int b = lane;
        float M = -CUDART_INF_F, Sm = 0.0f;
        for (int w2 = 0; w2 < kGSlots; ++w2)
          merge_partial(M, Sm, s_wm[w2 * kGMaxB + b], s_ws[w2 * kGMaxB + b], it2[b]);
        unsigned long long* r0 = rec.cta + (((size_t)par * B + b) * G + cta) * kGRecWords;
        st_rec(r0, __float_as_uint(M), seq);
        st_rec(r0 + 1, __float_as_uint(Sm), seq);
      }
      // While warp b polls, warp 2 + b turns this CTA's chunk partials of
      // request b into weights relative to the CTA's own max and their prefix
      // sums (fp64), so that the owner's chunk search is one rescale and one
      // ballot.
      if (gemv && cw >= 2 && cw - 2 < B) {
        const int b = cw - 2;
        float Acta = -CUDART_INF_F;
        for (int w2 = 0; w2 < kGSlots; ++w2) Acta = fmaxf(Acta, s_wm[w2 * kGMaxB + b]);
        const float2* lp = sPart + (size_t)b * part_cap;
        const int ca = 2 * lane, cb = ca + 1;
        const double wA = (ca < nc && lp[ca].y > 0.0f) ? partial_weight(lp[ca], Acta, it2[b]) : 0.0;
        const double wB = (cb < nc && lp[cb].y > 0.0f) ? partial_weight(lp[cb], Acta, it2[b]) : 0.0;
        const double pin = warp_incl_scan_d(wA + wB);
        s_cw[b * kGMaxChunks + ca] = wA;
        s_cw[b * kGMaxChunks + cb] = wB;
        s_cp[b * kGMaxChunks + ca] = pin - wB;
        s_cp[b * kGMaxChunks + cb] = pin;
        if (lane == 0) s_acta[b] = Acta;
      }
      // warp b: gathers the partials of request b from every CTA (level 1)
      float M = 0.0f;
      double Z = 0.0, T = 0.0, before = 0.0;
      int cstar = -1;
      if (gemv && cw < B) {
        const int b = cw;
        const unsigned long long* cr = rec.cta + (((size_t)par * B + b) * G) * kGRecWords;
        // one warp per CTA polls; a poll is one round of loads (no back-off: the
        // reads are a few KB per round across the grid)
        const int per = (G + 31) / 32;
        const int c0 = min(lane * per, G), c1 = min(c0 + per, G);
        float2 q[kGPerLane];
        unsigned pend = 0;
#pragma unroll
        for (int i = 0; i < kGPerLane; ++i) {
          q[i] = make_float2(-CUDART_INF_F, 0.0f);
          if (c0 + i < c1) pend |= 1u << i;
        }
        const uint64_t tstart = global_timer_ns();
        for (uint32_t polls = 1;; ++polls) {
          ulonglong2 m[kGPerLane];
#pragma unroll
          for (int i = 0; i < kGPerLane; ++i)
            if (pend & (1u << i)) m[i] = ld_rec2(cr + (size_t)kGRecWords * (c0 + i));
#pragma unroll
          for (int i = 0; i < kGPerLane; ++i) {
            // (a test skew makes the first position wait for a later one)
            const uint32_t want = seq + (k == 0 ? test_skew : 0u);
            if ((pend & (1u << i)) && (uint32_t)(m[i].x >> 32) == want && (uint32_t)(m[i].y >> 32) == want) {
              q[i] = make_float2(__uint_as_float((uint32_t)m[i].x), __uint_as_float((uint32_t)m[i].y));
              pend &= ~(1u << i);
            }
          }
          if (!__any_sync(0xffffffffu, pend != 0)) break;
          if (__any_sync(0xffffffffu, wait_expired(tstart, polls))) {
            if (lane == 0) {
              *s_abort = 1;
              raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
            }
            break;
          }
        }
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int i = 0; i < kGPerLane; ++i) mx = fmaxf(mx, q[i].x);
        M = warp_max(mx);
        double w[kGPerLane], wsum = 0.0;
#pragma unroll
        for (int i = 0; i < kGPerLane; ++i) {
          w[i] = partial_weight(q[i], M, it2[b]);
          wsum += w[i];
        }
        const double incl = warp_incl_scan_d(wsum);
        Z = __shfl_sync(0xffffffffu, incl, 31);
        T = (double)s_ud[b * K + k] * Z;
        double start = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) start = 0.0;
        const unsigned own = __ballot_sync(0xffffffffu, start <= T && T < incl && wsum > 0.0);
        int pick = -1, lastp = -1;
        double bef = start, lastb = start;
        {
          double cum = start;
#pragma unroll
          for (int i = 0; i < kGPerLane; ++i) {
            if (pick < 0 && w[i] > 0.0) {
              lastp = c0 + i;
              lastb = cum;
              if (cum + w[i] > T) {
                pick = c0 + i;
                bef = cum;
              }
            }
            cum += w[i];
          }
        }
        if (pick < 0) {
          pick = lastp;
          bef = lastb;
        }
        if (own) {
          const int ol = __ffs(own) - 1;
          cstar = __shfl_sync(0xffffffffu, pick, ol);
          before = __shfl_sync(0xffffffffu, bef, ol);
        } else {  // no crossing (u*Z rounded to Z): last CTA with mass
          const unsigned pos = __ballot_sync(0xffffffffu, lastp >= 0);
          const int pl = pos ? 31 - __clz(pos) : 0;
          cstar = __shfl_sync(0xffffffffu, lastp, pl);
          if (cstar < 0) cstar = 0;
          before = -CUDART_INF;
        }
      }
      gemv_sync();  // the chunk weights of every request are in shared memory
      // the CTA that holds the sample resolves chunk and token; scales: global
      // = f * (relative to the CTA max) and (relative to the CTA max) = g *
      // (relative to the chunk max)
      if (gemv && cw < B && cstar == cta) {
        const int b = cw;
        const float Acta = s_acta[b];
        const double f = (double)ex2((Acta - M) * it2[b]);
        const double Tp = (T - before) / f;
        const int ca = 2 * lane, cb = ca + 1;
        const double wA = s_cw[b * kGMaxChunks + ca], wB = s_cw[b * kGMaxChunks + cb];
        const double pA = s_cp[b * kGMaxChunks + ca], pB = s_cp[b * kGMaxChunks + cb];
        const bool hitA = wA > 0.0 && pA > Tp;
        const bool hitB = wB > 0.0 && pB > Tp;
        const unsigned h = __ballot_sync(0xffffffffu, hitA || hitB);
        int chunk;
        double before2;  // mass before the chunk, relative to the CTA max
        if (h) {
          const int hl = __ffs(h) - 1;
          chunk = __shfl_sync(0xffffffffu, hitA ? ca : cb, hl);
          before2 = __shfl_sync(0xffffffffu, hitA ? pA - wA : pB - wB, hl);
        } else {
          const unsigned hp = __ballot_sync(0xffffffffu, wA > 0.0 || wB > 0.0);
          const int hl = hp ? 31 - __clz(hp) : 0;
          chunk = __shfl_sync(0xffffffffu, (wB > 0.0) ? cb : ca, hl);
          if (!hp) chunk = 0;
          before2 = -CUDART_INF;
        }
        // the chunk's rows: weights relative to the chunk max, kept by the epilogue
        const double g = (double)ex2((sPart[(size_t)b * part_cap + chunk].x - Acta) * it2[b]);
        const double Tpp = (Tp - before2) / g;
        const int vl = chunk * kChunk + lane;
        const int v = v0 + vl;
        const bool valid = vl < nrows;
        const double e = valid ? (double)sBias[(size_t)b * rows_cap + vl] : 0.0;
        const int pl = pick_lane(e, 0.0, Tpp);
        const int x = __shfl_sync(0xffffffffu, valid ? v : 0, pl);
        // start pulling U[x] into L2 for every CTA's next position, publish
        // {position, token}, then write the outputs
        if (k + 1 < K && lane < (kGRank * 2) / 128)
          prefetch_l2(reinterpret_cast<const uint8_t*>(p.U + (size_t)x * kGRank) + lane * 128);
        if (lane == 0) st_rec(rec.tok + (size_t)b * kGRecWords, (uint32_t)x, seq);
        if (lane == pl) {
          const size_t o = (size_t)b * K + k;
          if (!(Z > 0.0) || !isfinite(Z)) {
            raise_flag(p.flags, DSPARK_FLAG_NONFINITE);
            p.tokens[o] = 0;
            p.p_tok[o] = 0.0f;
            p.lse[o] = CUDART_NAN_F;
            p.ref_max[o] = M;
            p.ref_sum[o] = 1.0f;
          } else {
            p.tokens[o] = x;
            p.p_tok[o] = (float)(f * g * e / Z);
            p.lse[o] = (float)((double)M * (double)itv[b] + log(Z));
            p.ref_max[o] = M;
            p.ref_sum[o] = (float)Z;
          }
        }
      }
      // one thread per request waits for the token; every warp then loads its U[x] slice
      // (after the last position nothing waits for it)
      if (cw == 0 && lane < B && k + 1 < K) {
        unsigned long long v;
        bool to = false;
        backoff_spin_u64(rec.tok + (size_t)lane * kGRecWords, seq, &v, &to);
        if (to) {
          *s_abort = 1;
          raise_flag(p.flags, DSPARK_FLAG_TIMEOUT);
        }
        s_i[1 + lane] = min(max((int)(uint32_t)v, 0), V - 1);
      }
      // every reader of sBase[buf], sBias and sPart for position k is past this barrier
      const bool abort = gemv_sync_or(*s_abort != 0);
      if (cw == 0 && lane == 0) mbar_arrive(&baseEmpty[buf]);  // buffer free for position k+2
      if (abort) break;
      if (k + 1 < K) {
        int x[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) x[b] = (b < B) ? s_i[1 + b] : -1;
        load_u_slice<NB>(p.U, x, B, lane, u);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kPTmemCols);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

inline bool persist_supported(int V, int r, int B) {
  if (B < 1 || B > kPMaxB || r % 64 != 0 || r < 64 || r > 256 || V % 4 != 0 || V < kTileN)
    return false;
  const PersistLayout L = persist_layout(V, r, B);
  if (gemv_path(r, B)) {
    int max_chunks, max_tiles;
    gemv_runs(n_chunks_of(V), L.G, &max_chunks, &max_tiles);
    if (max_chunks > kGMaxChunks) return false;
    return L.max_nt <= kPMaxTiles && L.n_stages >= 1;  // any ring depth is deadlock-free
  }
  return L.max_nt <= kPMaxTiles && L.n_stages >= kPMinStages;
}

template <typename Kern>
inline dspark_status persist_launch_kernel(Kern kern, int threads, const CUtensorMap& tm_w,
                                           const PersistArgs& a, const PersistLayout& L,
                                           cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.G);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = s;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tm_w, a) == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

inline dspark_status persist_launch(const CUtensorMap& tm_w, PersistArgs a, GemvRecs recs,
                                    cudaStream_t s) {
  static DeviceOnce once;
  once_per_device(once, [] {
    cudaFuncSetAttribute(draft_persist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kPSmemLimit);
    cudaFuncSetAttribute(draft_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kPSmemLimit);
    cudaFuncSetAttribute(draft_gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kPSmemLimit);
  });
  const PersistLayout L = persist_layout(a.V, a.r, a.B);
  a.max_nt = L.max_nt;
  a.n_stages = L.n_stages;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.G);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = s;
  cudaLaunchAttribute attrs[1];
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (gemv_path(a.r, a.B)) {
    cfg.blockDim = dim3(kGThreads);
    e = (a.B == 1) ? cudaLaunchKernelEx(&cfg, draft_gemv_kernel<1>, tm_w, a, recs)
                   : cudaLaunchKernelEx(&cfg, draft_gemv_kernel<2>, tm_w, a, recs);
  } else {
    cfg.blockDim = dim3(kPThreads);
    e = cudaLaunchKernelEx(&cfg, draft_persist_kernel, tm_w, a);
  }
  return e == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

// Bytes of the position records of the GEMV variant (zeroed by the caller
// before each call): CTA partials [2][B][G] and token words [B], one
// 128-byte line each.
inline size_t gemv_rec_words_cta(int B) { return (size_t)2 * B * kGMaxG * kGRecWords; }
inline size_t gemv_rec_bytes(int B) {
  return (gemv_rec_words_cta(B) + (size_t)B * kGRecWords) * 8;
}

}  // namespace dspark
