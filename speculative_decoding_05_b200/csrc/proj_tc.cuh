// proj_tc.cuh -- tensor-core (tcgen05) projection for large batches.
//
// bias[b, v] = U[x_b] . W[v] is a [B, r] x [r, V] GEMM once B is large.
// Each CTA owns a block of kBlockM = 128 requests (MMA M; rows past B are
// zero) and a contiguous range of vocabulary tiles of kTileN = 128 rows
// (MMA N); K = r (64..256).  The gathered U rows (operand A) are written to
// shared memory once per launch in the 128-byte-swizzled K-major layout,
// only as many rows as the block has requests (rounded up to 8): the MMA
// still reads 128 rows, and the ones past them fall on whatever bytes follow
// in shared memory.  Row m of the product depends on row m of A alone, so
// those rows only reach TMEM lanes of requests past the batch, which no
// epilogue warp reads;
// W tiles (operand B) stream through a TMA ring and the accumulator lives
// in TMEM (two 128-column buffers, so the epilogue of tile t overlaps the
// MMAs of tile t+1).  The epilogue thread of request b reads its TMEM row
// (tcgen05.ld) and reduces every 32-row chunk of its row to a softmax
// partial locally -- no cross-thread reduction, because the request is the
// TMEM lane.
//
// The draft launch carries programmatic stream serialisation: the next
// position's producers fill the rings while the sampler runs (see the
// grid_dep_wait below); the residual launch is plain.
//
//   warp 0       W producer (TMA, evict-last: W is re-read every position)
//   warp 1       TMEM allocator + MMA issuer (one thread)
//   warp 2       base-logit producer (TMA 3-D boxes, evict-first)   [draft]
//                target / base row-segment producer (TMA gather4)   [residual]
//   warps 3..10  epilogue: two warpgroups of 128 threads (= 128 requests);
//                warpgroup g takes the 32-column chunks g, g + 2 of every
//                tile
//
// Draft mode streams base[b, k, v0:v0+32] boxes through a second TMA ring.
// Residual mode needs the per-request rows target[row_b, :] and
// base[b, j_b, :] (j_b differs between requests): warp 2 fetches each
// request's 256-byte segment of every kResCols = 64 columns (two chunks)
// with TMA tile::gather4 loads (four rows of a one-row-high box per
// instruction) into a second ring, unswizzled (rows at a 256-byte stride);
// both warpgroups read every stage.  A gather through the
// load/store units instead (per-thread loads, or 16-byte cp.async copies)
// was capped near 5 GB/s per SM by the SM's outstanding misses.  The
// epilogue thread of request m reads its row's 16-byte chunks starting at
// chunk m & 7, so the eight lanes of a shared-memory phase meet eight
// different bank groups, and rotates its TMEM values to the same order.
#pragma once

#include <cudaTypedefs.h>

#include "proj_simt.cuh"
#include "tc_common.cuh"

namespace dspark {

constexpr int kBlockM = 128;
// Epilogue warpgroups (128 threads = 128 requests each), two chunks of every
// tile each.  Four warpgroups of one chunk each (608 threads) measured
// slower at B = 512 (0.127 against 0.102 ms per position): the register cap
// of the larger block spilled the 64 accumulator and base values.
template <bool kRes>
__host__ __device__ constexpr int tc_epi_groups() { return 2; }
template <bool kRes>
__host__ __device__ constexpr int tc_threads() { return 96 + 128 * tc_epi_groups<kRes>(); }
constexpr int kTileN = 128;
// Columns of one residual stage: two 32-column chunks, so each gather4 load
// moves four 256-byte row segments (the loads' issue rate bounds the mode).
constexpr int kResCols = 64;
constexpr int kWStagesMax = 12;     // W ring depth: as deep as shared memory allows
constexpr int kBStagesMax = 16;     // base ring depth (draft): likewise
constexpr int kStageBytes = 16384;  // 128 rows x 128 bytes
constexpr size_t kTcSmemLimit = 232448 - 1024;  // dynamic: 227 KB less the static arrays
constexpr int kTmemCols = 512;     // two 128-column accumulators, then operand A
constexpr uint32_t kACol = 256;    // operand A's first column (ra / 2 columns)

struct TcPlan {
  CUtensorMap tm_w;
  CUtensorMap tm_base;  // draft: [B, K, V] boxes; residual: [B * K, V] rows
  CUtensorMap tm_tgt;   // residual: target rows [n_rows, V]
  const float* base;
  const float* target;
  const __nv_bfloat16* U;
  int V, r, B, K;
  int n_tiles, n_bb, ctas_per_bb;
  int w_stages, b_stages, base_rows;  // ring depths, request rows per base box
  int w_group;                        // W k-blocks per ring stage
  const __nv_bfloat16* a_rows;        // draft: per-request A rows (split state) or NULL
  int a_split;                         // 1: a_rows hold 2r columns (high, low halves)
};

// Request rows of a base-logit box: the batch rounded up to 8 (the 128-byte
// swizzle repeats every 8 rows), at most one block of kBlockM.  A batch of 64
// then moves half the bytes of a full 128-row box.
inline int tc_base_rows(int B) { return B < kBlockM ? (B + 7) / 8 * 8 : kBlockM; }
// Bytes of one k-block of operand A (and of one base box): the block's
// request rows, 128 bytes each.  A multiple of 1024, the swizzle atom.
inline size_t tc_a_stage_bytes(int B) { return (size_t)tc_base_rows(B) * 128; }
// One stage of the second ring: the base box of a 32-column chunk (draft),
// or the target and base segments of kResCols columns of every request
// (residual).
inline size_t tc_r_stage_bytes(int B, bool residual) {
  return residual ? (size_t)2 * tc_base_rows(B) * kResCols * 4 : tc_a_stage_bytes(B);
}
// Stages of the second ring per tile.
inline int tc_r_stages_per_tile(bool residual) { return residual ? kTileN / kResCols : kTileN / 32; }
// Alignment slack and the barriers (operand A lives in tensor memory).
inline size_t tc_fixed_bytes(int ra, int B, bool residual) {
  (void)ra;
  (void)B;
  (void)residual;
  return 1024 + 512;
}
// Ring depths.  Each copy in flight waits about the same time for its
// bytes, so the two rings share what is left in proportion to what they
// move per tile: W r / 64 stages of 16 KB, the second ring kTileN / 32
// stages.  The second ring's depth is even: chunk parity picks the epilogue
// warpgroup, so every stage is then read by one warpgroup only, which waits
// on each fill of it in turn.  (With an odd depth a stage alternates between
// the warpgroups, and a parity wait on fill f can pass while fill f - 1,
// meant for the other warpgroup, is still landing: the waiter would read the
// wrong chunk and release the stage early.)  W takes what is left, at least
// two stages (a ring shorter than a tile still flows: the MMAs free its
// stages in order).
inline int tc_b_stages(int r, int B, bool residual, int a_split = 0) {
  const size_t ring = kTcSmemLimit - tc_fixed_bytes(r << a_split, B, residual);
  const size_t w_tile = (size_t)(r / 64) * kStageBytes;
  const size_t rstage = tc_r_stage_bytes(B, residual);
  const size_t b_tile = (size_t)tc_r_stages_per_tile(residual) * rstage;
  int s = (int)(ring * b_tile / (w_tile + b_tile) / rstage);
  if (s < 2) s = 2;
  while (s > 2 && ring < (size_t)s * rstage + 2 * kStageBytes) --s;
  if (s > kBStagesMax) s = kBStagesMax;
  return s & ~1;
}
inline int tc_w_stages(int r, int B, bool residual, int a_split = 0) {
  const size_t ring = kTcSmemLimit - tc_fixed_bytes(r << a_split, B, residual);
  const size_t left = ring - (size_t)tc_b_stages(r, B, residual, a_split) * tc_r_stage_bytes(B, residual);
  int s = (int)(left / kStageBytes);
  if (s > kWStagesMax) s = kWStagesMax;
  return s;
}
inline size_t tc_smem_bytes(int r, int B, bool residual, int a_split = 0) {
  return tc_fixed_bytes(r << a_split, B, residual) +
         (size_t)tc_w_stages(r, B, residual, a_split) * kStageBytes +
         (size_t)tc_b_stages(r, B, residual, a_split) * tc_r_stage_bytes(B, residual);
}

inline bool tc_supported(int V, int r, int B) {
  return B > 16 && r % 64 == 0 && r >= 64 && r <= 256 && V % 4 == 0 && V >= kTileN;
}

template <bool kRes>
__global__ void __launch_bounds__(tc_threads<kRes>(), 1)
proj_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_base,
               const __grid_constant__ CUtensorMap tm_tgt, const __nv_bfloat16* __restrict__ U, int V, int r, int B, int K, int k,
               const int32_t* __restrict__ prev_token, const int32_t* __restrict__ tokens,
               const float* __restrict__ inv_temp, const float* __restrict__ target,
               const float* __restrict__ base, const ResInfo* __restrict__ info,
               float* __restrict__ draft_logits, float* __restrict__ draft_bias,
               float2* __restrict__ part, float2* __restrict__ cta_part, int n_chunks,
               int n_tiles, int ctas_per_bb, int n_ws, int n_bs, int base_rows,
               const __nv_bfloat16* __restrict__ a_rows, int a_split, int w_group,
               unsigned* flags) {
  // n_ws: W ring space in 16 KB k-block units; w_group: k-blocks per ring
  // stage (one barrier pair, one commit), so the ring has n_ws / w_group stages
  constexpr int kEpi = tc_epi_groups<kRes>();
  constexpr int kCpg = (kTileN / 32) / kEpi;  // chunks of a tile per epilogue warpgroup
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nkb = r >> 6;
  // operand A: U[x] (r columns), or with a_rows (draft only) the request's
  // row of a_rows, r << a_split columns: a state split into bf16 high and
  // low parts, both multiplied by the same W block and accumulated
  const int ra = r << a_split;
  const int bstage = base_rows * 128;  // bytes of one base box
  uint8_t* sW = sm;
  uint8_t* sBase = sW + n_ws * kStageBytes;
  // one stage of the second ring; residual: target segments, then (at
  // bhalf) base segments, kResCols columns of each request at a 256-byte stride
  const int bhalf = base_rows * kResCols * 4;
  const int rstage = kRes ? 2 * bhalf : bstage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sBase + n_bs * rstage);
  uint64_t* fullW = bars;
  uint64_t* emptyW = fullW + kWStagesMax;
  uint64_t* fullB = emptyW + kWStagesMax;
  uint64_t* emptyB = fullB + kBStagesMax;
  uint64_t* accFull = emptyB + kBStagesMax;
  uint64_t* accEmpty = accFull + 2;
  uint64_t* mmaDrain = accEmpty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mmaDrain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bb = blockIdx.x / ctas_per_bb, pi = blockIdx.x % ctas_per_bb;
  const int t0 = (int)((long long)pi * n_tiles / ctas_per_bb);
  const int t1 = (int)((long long)(pi + 1) * n_tiles / ctas_per_bb);
  const int nt = t1 - t0;
  // Odd draft positions walk the range backwards, so a position starts on
  // the W tiles the one before it read last (the likeliest still in L2).
  const bool rev = !kRes && (k & 1);
  auto tile_at = [&](int i) { return rev ? t1 - 1 - i : t0 + i; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < n_ws; ++i) {
      mbar_init(&fullW[i], 1);
      mbar_init(&emptyW[i], 1);
    }
    for (int i = 0; i < n_bs; ++i) {
      mbar_init(&fullB[i], 1);
      // draft: the four warps of the chunk's warpgroup; residual: a stage
      // holds one chunk of each warpgroup
      mbar_init(&emptyB[i], kRes ? 4 * kEpi : 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accFull[i], 1);
      mbar_init(&accEmpty[i], 4 * kEpi);
    }
    mbar_init(mmaDrain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // The draft projection is launched with a programmatic dependency on the
  // kernel before it (the previous position's sampler).  Every warp that
  // reads what that kernel wrote (tokens, operand rows) or writes what it
  // reads (the partials) waits for it here; the producers read only W and
  // the base logits, which no kernel of the call writes, so from position 1
  // on they start filling the rings at once.
  if (warp == 1 || warp >= 3 || k == 0) grid_dep_wait();

  // operand A -> tensor memory, written by the epilogue warps: lane = the
  // request's row m, 32-bit column kACol + c holds the bf16 pair (2c, 2c + 1)
  // of U[x_m] (or of its a_rows row); rows past the batch are zero.  A warp
  // reaches only its lane quarter, so each warpgroup covers all 128 rows and
  // takes every other 64-element unit of them; a lane loads and stores its
  // units, 8 16-byte pieces per unit.  The MMA warp joins the barrier that
  // ends the writes.
  constexpr int kGather = tc_threads<kRes>() - 64;  // warp 1 + the epilogue warps
  if (warp >= 3) {
    const int eg = (warp - 3) >> 2;
    const int m = (warp & 3) * 32 + lane;
    const int b = bb * kBlockM + m;
    int x = -1;
    if (b < B) {
      if (kRes) {
        const ResInfo& ri = info[b];
        x = ri.bonus ? -1 : ri.x_prev;
      } else if (a_rows != nullptr) {
        x = b;
      } else {
        // volatile loads (__ldcg), kept behind grid_dep_wait: the token of
        // position k - 1 comes from the sampler this launch overlaps
        x = (k == 0) ? __ldcg(prev_token + b) : __ldcg(tokens + (size_t)b * K + (k - 1));
        if (x >= V || (k > 0 && x < 0)) {
          raise_flag(flags, DSPARK_FLAG_BAD_TOKEN);
          x = (k > 0) ? (x < 0 ? 0 : V - 1) : -1;
        }
      }
    }
    const __nv_bfloat16* src = a_rows != nullptr ? a_rows : U;
    const uint4* row = reinterpret_cast<const uint4*>(src + (size_t)(x < 0 ? 0 : x) * ra);
    const uint32_t lanes = tmem + ((uint32_t)((warp & 3) * 32) << 16) + kACol;
    const int units = ra >> 6;  // 64 elements = 32 columns each
    for (int u = eg; u < units; u += kEpi) {
      uint32_t regs[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint4 val = make_uint4(0, 0, 0, 0);
        if (x >= 0) val = __ldg(row + u * 8 + q);
        regs[4 * q] = val.x;
        regs[4 * q + 1] = val.y;
        regs[4 * q + 2] = val.z;
        regs[4 * q + 3] = val.w;
      }
      tmem_st32(lanes + (uint32_t)(u * 32), regs);
    }
    tmem_st_wait();
  }
  if (warp == 1 || warp >= 3) {
    tc_fence_before();
    named_sync(1, kGather);
  }

  if (warp == 0) {
    // ---------------- W producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int it = 0;
      const int ngrp = (nkb + w_group - 1) / w_group, nslot = n_ws / w_group;
      for (int i = 0; i < nt && !*s_abort; ++i) {
        const int t = tile_at(i);
        for (int g = 0; g < ngrp; ++g, ++it) {
          const int s = it % nslot;
          const uint32_t ph = (uint32_t)(it / nslot) & 1u;
          if (!mbar_wait(&emptyW[s], ph ^ 1u)) {
            *s_abort = 1;
            raise_flag(flags, DSPARK_FLAG_TIMEOUT);
            break;
          }
          const int nk = min(w_group, nkb - g * w_group);
          mbar_arrive_expect_tx(&fullW[s], (uint32_t)(nk * kStageBytes));
          for (int h = 0; h < nk; ++h)
            tma_load_2d_hint(sW + (s * w_group + h) * kStageBytes, &tm_w, &fullW[s],
                             (g * w_group + h) * 64, t * kTileN, pol);
        }
      }
      // Tail: a stage is released by a commit of the MMAs that read it, an
      // arrive the tensor core makes on this CTA's barrier when they
      // complete.  Wait for the releases of the last stages filled, so the
      // CTA never exits with such an arrive still in flight; after an abort,
      // wait for the copies still in flight instead.
      if (!*s_abort) wait_ring_released(emptyW, nslot, it, flags);
      else drain_ring_loads(fullW, nslot, it);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kBlockM, kTileN);
      const uint32_t aT = tmem + kACol, w0 = smem_u32(sW);
      const int ngrp = (nkb + w_group - 1) / w_group, nslot = n_ws / w_group;
      int it = 0;
      for (int i = 0; i < nt && !*s_abort; ++i) {
        const int a = i & 1;
        const uint32_t aph = (uint32_t)(i >> 1) & 1u;
        if (!mbar_wait(&accEmpty[a], aph ^ 1u)) {
          *s_abort = 1;
          raise_flag(flags, DSPARK_FLAG_TIMEOUT);
          break;
        }
        tc_fence_after();
        bool ok = true;
        for (int g = 0; g < ngrp; ++g, ++it) {
          const int s = it % nslot;
          const uint32_t ph = (uint32_t)(it / nslot) & 1u;
          if (!mbar_wait(&fullW[s], ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(w_group, nkb - g * w_group);
          for (int hk = 0; hk < nk; ++hk) {
            const int kb = g * w_group + hk;
            for (int h = 0; h <= a_split; ++h) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bd = sdesc_sw128(w0 + (s * w_group + hk) * kStageBytes + kk * 32);
                mma_bf16_ts(tmem + a * kTileN, aT + (uint32_t)(((h * nkb + kb) * 4 + kk) * 8), bd,
                            idesc, (kb | kk | h) != 0);
              }
            }
          }
          mma_commit(&emptyW[s]);
        }
        if (!ok) {
          *s_abort = 1;
          raise_flag(flags, DSPARK_FLAG_TIMEOUT);
          break;
        }
        mma_commit(&accFull[a]);
      }
      drain_mma(mmaDrain);
    }
  } else if (warp == 2 && kRes) {
    // ---------------- target / base row producer (residual)
    // lane g gathers requests 4g..4g+3: their target rows and base rows
    // (row 0 stands in for a request past the batch, or for the base row of
    // a bonus request; neither is read)
    const int groups = base_rows >> 2;
    int trow[4] = {0, 0, 0, 0}, brow[4] = {0, 0, 0, 0};
    if (lane < groups) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int b = bb * kBlockM + 4 * lane + i;
        if (b < B) {
          const ResInfo& ri = info[b];
          trow[i] = (int)ri.row;
          if (!ri.bonus) brow[i] = b * K + ri.j;
        }
      }
    }
    const uint64_t pol = policy_evict_first();
    int it = 0;
    for (int i = 0; i < nt && !*s_abort; ++i) {
      const int t = tile_at(i);
      bool ok = true;
      for (int cs = 0; cs < kTileN / kResCols; ++cs, ++it) {
        const int s = it % n_bs;
        const uint32_t ph = (uint32_t)(it / n_bs) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&emptyB[s], ph ^ 1u))) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(&fullB[s], (uint32_t)(2 * groups * 4 * kResCols * 4));
        __syncwarp();
        if (lane < groups) {
          const int v0 = t * kTileN + cs * kResCols;
          uint8_t* st = sBase + s * rstage + lane * (4 * kResCols * 4);
          tma_gather4_hint(st, &tm_tgt, &fullB[s], v0, trow[0], trow[1], trow[2], trow[3], pol);
          tma_gather4_hint(st + bhalf, &tm_base, &fullB[s], v0, brow[0], brow[1], brow[2], brow[3],
                           pol);
        }
      }
      if (!ok) {
        *s_abort = 1;
        raise_flag(flags, DSPARK_FLAG_TIMEOUT);
        break;
      }
    }
    if (*s_abort && lane == 0) drain_ring_loads(fullB, n_bs, it);
  } else if (warp == 2) {
    // ---------------- base-logit producer (draft only)
    if (!kRes && lane == 0) {
      const uint64_t pol = policy_evict_first();
      int it = 0;
      for (int i = 0; i < nt && !*s_abort; ++i) {
        const int t = tile_at(i);
        for (int cb = 0; cb < kTileN / 32; ++cb, ++it) {
          const int s = it % n_bs;
          const uint32_t ph = (uint32_t)(it / n_bs) & 1u;
          if (!mbar_wait(&emptyB[s], ph ^ 1u)) {
            *s_abort = 1;
            raise_flag(flags, DSPARK_FLAG_TIMEOUT);
            break;
          }
          mbar_arrive_expect_tx(&fullB[s], (uint32_t)bstage);
          tma_load_3d_hint(sBase + s * bstage, &tm_base, &fullB[s], t * kTileN + cb * 32, k,
                           bb * kBlockM, pol);
        }
      }
      if (*s_abort) drain_ring_loads(fullB, n_bs, it);
    }
  } else {
    // ---------------- epilogue: thread = request (TMEM lane)
    // warpgroup eg takes chunks eg, eg + kEpi, ... of every tile: chunk
    // parity picks the warpgroup, so with an even depth every stage of the
    // second ring is always read by the same warpgroup (see tc_b_stages)
    const int eg = (warp - 3) >> 2;
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;
    const int b = bb * kBlockM + m;
    const bool bval = b < B;
    // a warp whose 32 requests are all past the batch only keeps the
    // pipeline moving (its arrivals), without loading or reducing anything
    const bool wval = bb * kBlockM + quarter * 32 < B;
    const float it = bval ? checked_inv_temp(inv_temp, b, flags) : 1.0f;
    const float it2 = it * kLog2e;
    ResInfo ri{};
    if (kRes && bval) ri = info[b];
    // draft: this warpgroup's partial over all of its chunks of the range
    float Mr = -CUDART_INF_F, Sr = 0.0f;
    for (int i = 0; i < nt; ++i) {
      const int t = tile_at(i);
      const int a = i & 1;
      const uint32_t aph = (uint32_t)(i >> 1) & 1u;
      if (*s_abort || !mbar_wait(&accFull[a], aph)) {
        *s_abort = 1;
        raise_flag(flags, DSPARK_FLAG_TIMEOUT);
        break;
      }
      tc_fence_after();
      float2 pp[kCpg];
      if constexpr (!kRes) {
        // ---- draft: softmax partial of every 32-row chunk of the tile
#pragma unroll 1
        for (int ci = 0; ci < kCpg; ++ci) {
          const int cb = eg + kEpi * ci;
          float d[32];
          if (wval) tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + a * kTileN + cb * 32, d);
          float bv[32];
          const int v0 = t * kTileN + cb * 32;
          const int itB = i * (kTileN / 32) + cb;
          const int s = itB % n_bs;
          const uint32_t ph = (uint32_t)(itB / n_bs) & 1u;
          if (!mbar_wait(&fullB[s], ph)) {
            *s_abort = 1;
            raise_flag(flags, DSPARK_FLAG_TIMEOUT);
          }
          // a box holds base_rows requests: rows past it are not read (their
          // results are discarded, since base_rows >= the block's requests)
          const uint8_t* row = sBase + s * bstage + m * 128;
          if (wval) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float4 q4 = make_float4(0.f, 0.f, 0.f, 0.f);
              if (m < base_rows) q4 = *reinterpret_cast<const float4*>(row + ((j ^ (m & 7)) << 4));
              bv[4 * j] = q4.x; bv[4 * j + 1] = q4.y; bv[4 * j + 2] = q4.z; bv[4 * j + 3] = q4.w;
            }
          }
          float2 cpv = make_float2(-CUDART_INF_F, 0.0f);
          if (wval) {
            if (v0 + 32 > V) {
              // the ragged end of the vocabulary: rows past V carry no mass
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (v0 + j >= V) {
                  bv[j] = -CUDART_INF_F;
                  d[j] = 0.0f;
                }
            }
            cpv = chunk_partial32(bv, d, it2);
          }
          // the stage is released only once every lane's reads have returned
          consumed(cpv.x);
          consumed(cpv.y);
          __syncwarp();
          if (lane == 0) mbar_arrive(&emptyB[s]);
          if (!wval) continue;
          pp[ci] = cpv;
          merge_partial(Mr, Sr, pp[ci].x, pp[ci].y, it2);
          if (draft_bias != nullptr && bval) {
            float* dst = draft_bias + ((size_t)b * K + k) * (size_t)V + v0;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              if (v0 + j < V)
                *reinterpret_cast<float4*>(dst + j) = make_float4(d[j], d[j + 1], d[j + 2], d[j + 3]);
          }
          if (draft_logits != nullptr && bval) {
            float* dst = draft_logits + ((size_t)b * K + k) * (size_t)V + v0;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              if (v0 + j < V)
                *reinterpret_cast<float4*>(dst + j) =
                    make_float4((bv[j] + d[j]) * it, (bv[j + 1] + d[j + 1]) * it,
                                (bv[j + 2] + d[j + 2]) * it, (bv[j + 3] + d[j + 3]) * it);
          }
        }
      } else {
        // ---- residual: sums of max(0, p_t - p_d) and of p_t per chunk
#pragma unroll 1
        for (int ci = 0; ci < kCpg; ++ci) {
          const int cb = eg + kEpi * ci;
          float d[32], bv[32];
          if (wval) tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + a * kTileN + cb * 32, d);
          const int v0 = t * kTileN + cb * 32;
          const int itB = i * (kTileN / kResCols) + cb / (kResCols / 32);
          const int s = itB % n_bs;
          const uint32_t ph = (uint32_t)(itB / n_bs) & 1u;
          if (!mbar_wait(&fullB[s], ph)) {
            *s_abort = 1;
            raise_flag(flags, DSPARK_FLAG_TIMEOUT);
          }
          // this request's segments, staged by warp 2 (m < base_rows when
          // bval): slot j holds chunk (j + rot) & 7, and the TMEM values are
          // rotated to match (three select stages, static register indices).
          // Rows sit at a 256-byte stride, so the rotation still sends the
          // eight lanes of a shared-memory phase to eight bank groups.
          const int rot = lane & 7;
          float tq[32], dr[32];
          if (bval) {
#pragma unroll
            for (int x = 0; x < 32; ++x) dr[x] = (rot & 1) ? d[(x + 4) & 31] : d[x];
#pragma unroll
            for (int x = 0; x < 32; ++x) d[x] = (rot & 2) ? dr[(x + 8) & 31] : dr[x];
#pragma unroll
            for (int x = 0; x < 32; ++x) dr[x] = (rot & 4) ? d[(x + 16) & 31] : d[x];
            const uint8_t* trow = sBase + s * rstage + m * (kResCols * 4) + (cb % (kResCols / 32)) * 128;
            const uint8_t* brow = trow + bhalf;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int c = (j + rot) & 7;
              float4 t4 = make_float4(0.f, 0.f, 0.f, 0.f), b4 = t4;
              if (v0 + 4 * c < V) {
                t4 = *reinterpret_cast<const float4*>(trow + c * 16);
                if (!ri.bonus) b4 = *reinterpret_cast<const float4*>(brow + c * 16);
              }
              tq[4 * j] = t4.x; tq[4 * j + 1] = t4.y; tq[4 * j + 2] = t4.z; tq[4 * j + 3] = t4.w;
              bv[4 * j] = b4.x; bv[4 * j + 1] = b4.y; bv[4 * j + 2] = b4.z; bv[4 * j + 3] = b4.w;
            }
          }
          float qs4[4] = {0.0f, 0.0f, 0.0f, 0.0f}, ps4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          if (bval) {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
              if (v0 + 4 * ((x / 4 + rot) & 7) < V) {
                float pt;
                qs4[x & 3] += residual_q(tq[x], bv[x], dr[x], ri, it2, &pt);
                ps4[x & 3] += pt;
              }
            }
          }
          pp[ci] = make_float2((qs4[0] + qs4[1]) + (qs4[2] + qs4[3]), (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]));
          consumed(pp[ci].x);
          consumed(pp[ci].y);
          __syncwarp();
          if (lane == 0) mbar_arrive(&emptyB[s]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accEmpty[a]);
      if (bval && part != nullptr) {
        float2* dst = part + (size_t)b * n_chunks;
#pragma unroll
        for (int ci = 0; ci < kCpg; ++ci) {
          const int c = t * (kTileN / 32) + eg + kEpi * ci;
          if (c < n_chunks) dst[c] = pp[ci];
        }
      }
    }
    if (!kRes && bval && cta_part != nullptr)
      cta_part[((size_t)b * ctas_per_bb + pi) * kEpi + eg] = make_float2(Mr, Sr);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  // a driver entry point: the same for every device; looked up once,
  // thread-safe (function-local static)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
  }();
  return fn;
}

// SM count of the current device, looked up once per device.
inline int num_sms() {
  static DeviceOnce once;
  static int n[kMaxDevices];
  const int dev = current_device();
  int v = 0;
  if (dev >= 0 && dev < kMaxDevices) {
    std::call_once(once[dev], [&] {
      int c = 0;
      if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) c = 0;
      n[dev] = c > 0 ? c : 148;
    });
    v = n[dev];
  } else if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    v = 0;
  }
  return v > 0 ? v : 148;
}

// W [V, r] bf16 as 64 x 128 boxes (128-byte rows), 128-byte swizzle.
inline bool encode_w_map(CUtensorMap* m, const void* W, int V, int r) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)r, (cuuint64_t)V};
  cuuint64_t strides[1] = {(cuuint64_t)r * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kTileN};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// rows [n, V] fp32 as kResCols x 1 boxes (one row's 256-byte segment), no
// swizzle: the box of a tile::gather4 load, which takes four rows at once.
inline bool encode_rows_map(CUtensorMap* m, const float* p, int V, long long rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)V, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)V * 4};
  cuuint32_t box[2] = {(cuuint32_t)kResCols, 1};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// base [B, K, V] fp32 as 32 (v) x 1 (k) x 128 (b) boxes, 128-byte swizzle.
inline bool encode_base_map(CUtensorMap* m, const float* base, int V, int K, int B) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)V, (cuuint64_t)K, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)V * 4, (cuuint64_t)K * V * 4};
  cuuint32_t box[3] = {32, 1, (cuuint32_t)tc_base_rows(B)};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// k-blocks per W ring stage: a whole tile's (one wait and one commit per
// tile in the MMA thread, which issues every MMA and commit of the CTA:
// 1, 2 and 4 k-blocks per stage measured 1.61, 1.57 and 1.56 ms for the
// stress draft), halved until the ring still holds two stages.
inline int tc_w_group(int r, int w_units) {
  int g = r / 64;
  while (g > 1 && w_units / g < 2) g = (g + 1) / 2;
  return g;
}

// CTAs per request block, at most this many (the workspace holds this many
// partials per request and epilogue warpgroup).
constexpr int kTcMaxCtasPerBlock = 256;

inline void tc_grid(TcPlan& p) {
  p.n_tiles = (p.V + kTileN - 1) / kTileN;
  p.n_bb = (p.B + kBlockM - 1) / kBlockM;
  int per = num_sms() / p.n_bb;
  if (per < 1) per = 1;
  if (per > p.n_tiles) per = p.n_tiles;
  if (per > kTcMaxCtasPerBlock) per = kTcMaxCtasPerBlock;
  p.ctas_per_bb = per;
}

inline dspark_status tc_plan_draft(TcPlan& p, const float* base, const void* U, const void* W,
                                   int V, int r, int B, int K,
                                   const __nv_bfloat16* a_rows = nullptr) {
  p.V = V; p.r = r; p.B = B; p.K = K;
  p.a_rows = a_rows;
  p.a_split = a_rows != nullptr ? 1 : 0;
  p.base = base;
  p.target = nullptr;
  p.U = static_cast<const __nv_bfloat16*>(U);
  if (!encode_w_map(&p.tm_w, W, V, r) || !encode_base_map(&p.tm_base, base, V, K, B))
    return DSPARK_ERR_CUDA;
  p.tm_tgt = p.tm_w;  // unused in draft mode
  tc_grid(p);
  p.w_stages = tc_w_stages(r, B, false, p.a_split);
  p.b_stages = tc_b_stages(r, B, false, p.a_split);
  p.w_group = tc_w_group(r, p.w_stages);
  p.base_rows = tc_base_rows(B);
  return DSPARK_OK;
}

inline dspark_status tc_plan_residual(TcPlan& p, const float* target, long long n_rows,
                                      const float* base, const void* U, const void* W, int V,
                                      int r, int B, int K) {
  p.V = V; p.r = r; p.B = B; p.K = K;
  p.a_rows = nullptr;
  p.a_split = 0;
  p.base = base;
  p.target = target;
  p.U = static_cast<const __nv_bfloat16*>(U);
  if (!encode_w_map(&p.tm_w, W, V, r) || !encode_rows_map(&p.tm_tgt, target, V, n_rows) ||
      !encode_rows_map(&p.tm_base, base, V, (long long)B * K))
    return DSPARK_ERR_CUDA;
  tc_grid(p);
  p.w_stages = tc_w_stages(r, B, true);
  p.b_stages = tc_b_stages(r, B, true);
  p.w_group = tc_w_group(r, p.w_stages);
  p.base_rows = tc_base_rows(B);
  return DSPARK_OK;
}

template <bool kRes>
inline void tc_set_attr() {
  static DeviceOnce once;
  set_smem_once(once, proj_tc_kernel<kRes>, (int)kTcSmemLimit);
}

// The draft projection, launched with programmatic stream serialisation: it
// may start while the kernel before it (the sampler) runs, and orders
// itself behind it with griddepcontrol.wait.
inline void tc_launch_draft(const TcPlan& p, int k, const int32_t* prev, const int32_t* tokens,
                            const float* it, float* dl, float* dbias, float2* part,
                            float2* cta_part, unsigned* flags, cudaStream_t s) {
  tc_set_attr<false>();
  launch_dependent(proj_tc_kernel<false>, dim3(p.n_bb * p.ctas_per_bb), dim3(tc_threads<false>()),
                   tc_smem_bytes(p.r, p.B, false, p.a_split), s, p.tm_w, p.tm_base, p.tm_tgt, p.U,
                   p.V, p.r, p.B, p.K, k, prev, tokens, it, (const float*)nullptr, p.base,
                   (const ResInfo*)nullptr, dl, dbias, part, cta_part, n_chunks_of(p.V),
                   p.n_tiles, p.ctas_per_bb, p.w_stages, p.b_stages, p.base_rows, p.a_rows,
                   p.a_split, p.w_group, flags);
}

inline void tc_launch_residual(const TcPlan& p, const ResInfo* info, const float* it,
                               float2* rpart, unsigned* flags, cudaStream_t s) {
  tc_set_attr<true>();
  proj_tc_kernel<true><<<p.n_bb * p.ctas_per_bb, tc_threads<true>(), tc_smem_bytes(p.r, p.B, true),
                         s>>>(p.tm_w, p.tm_base, p.tm_tgt, p.U, p.V, p.r, p.B, p.K, 0, nullptr,
                              nullptr, it, p.target, p.base, info, nullptr, nullptr, rpart,
                              nullptr, n_chunks_of(p.V), p.n_tiles, p.ctas_per_bb, p.w_stages,
                              p.b_stages, p.base_rows, (const __nv_bfloat16*)nullptr, 0,
                              p.w_group, flags);
}

}  // namespace dspark
