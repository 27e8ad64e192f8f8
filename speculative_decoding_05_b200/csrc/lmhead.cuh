// lmhead.cuh -- the verify with the target logits formed on chip from the
// target model's final hidden states and its LM head.
//
// freeaitool.com, "DeepSeek DSpark complete guide", 6.3: the draft's
// training receives the target model's last hidden state and projects it
// through the LM head locally, so the vocabulary-sized rows never travel.
// Here the same projection feeds the verify's flattened, variable-length
// rows (yage.ai, "DSpark speculative decoding hardware scheduling",
// variable-length verify paragraph): the logit row of a verified position
// is hidden[row] . E[v] for every v, E the head [V, dm], and it is reduced
// on chip instead of being read from memory.
//
// lmhead_tc_kernel is a tcgen05 GEMM D = H . E^T over 128-row blocks of H
// (MMA M, TMEM lanes) and 128-row tiles of E (MMA N), K = dm streamed in
// 64-wide blocks: both operands arrive by TMA (128-byte swizzle, K-major)
// into one ring whose stage holds an H block and an E block.  Each CTA owns
// a contiguous range of E tiles and walks, for every tile, all row blocks
// of the launch, so E is read from memory once per launch and H (small)
// from L2.  Accumulators: two 128-column TMEM buffers, so the epilogue of
// one unit overlaps the MMAs of the next.  Epilogues:
//   kLhStats   per verified row, the CTA's softmax partial (max of the raw
//              logits, sum of exp((l - max) / T)) over its vocabulary range,
//              in the layout of the verify's target-row partials, and the
//              raw logit of the row's drafted token;
//   kLhLogits  the raw logits of the rows (the verify's one correction /
//              bonus row per request) to a scratch matrix.
//
//   warp 0      producer (TMA)
//   warp 1      TMEM allocator + MMA issuer (one thread)
//   warps 2..5  epilogue: thread = row of the block (TMEM lane)
#pragma once

#include "proj_tc.cuh"

namespace dspark {

constexpr int kLhThreads = 192;
constexpr int kLhStage = 2 * kStageBytes;  // one H block and one E block
constexpr int kLhMaxStages = 6;
constexpr int kLhMaxBlocks = 16;           // row blocks of one launch (2048 rows)
constexpr int kLhTmemCols = 256;
constexpr int kLhStats = 0, kLhLogits = 1;

// Dynamic shared memory: alignment slack, the ring, the per-row partials of
// the row blocks (stats), the barriers.
inline size_t lh_smem_bytes() {
  return 1024 + (size_t)kLhMaxStages * kLhStage + (size_t)kLhMaxBlocks * 128 * sizeof(float2) +
         512;
}

struct LhArgs {
  int n_rows;       // rows of H in this launch (row r of H is hidden row row0 + r)
  long long row0;   // first hidden row of the launch (stats) / 0 (logits)
  int dm, V, n_tiles, n_blocks;
  // stats
  const int* row_req;   // [total rows] request of each hidden row, -1: not verified
  const int* row_pos;   // [total rows] its position p (0..L_b)
  const float* inv_temp;
  const int32_t* tokens;  // [B, K] drafted tokens
  const int32_t* verify_len;
  int K;
  float2* tpart;        // [B * (K + 1)][G]
  float* tok_logit;     // [total rows]
  // logits
  float* logits;        // [n_rows, V]
  unsigned* flags;
};

template <int kMode>
__global__ void __launch_bounds__(kLhThreads, 1)
lmhead_tc_kernel(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_e,
                 const LhArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = sm;
  float2* spart = reinterpret_cast<float2*>(ring + kLhMaxStages * kLhStage);  // [blocks][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(spart + kLhMaxBlocks * 128);
  uint64_t* full = bars;
  uint64_t* empty = full + kLhMaxStages;
  uint64_t* accFull = empty + kLhMaxStages;
  uint64_t* accEmpty = accFull + 2;
  uint64_t* mmaDrain = accEmpty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mmaDrain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const int t0 = (int)((long long)g * a.n_tiles / G), t1 = (int)((long long)(g + 1) * a.n_tiles / G);
  const int n_units = (t1 - t0) * a.n_blocks;
  const int nkb = a.dm >> 6;
  constexpr int S = kLhMaxStages;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accFull[i], 1);
      mbar_init(&accEmpty[i], 4);
    }
    mbar_init(mmaDrain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kLhTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer: H block and E block of every k step
    if (lane == 0) {
      const uint64_t ph_ = policy_evict_last();  // H: re-read for every tile
      int it = 0;
      for (int u = 0; u < n_units && !*s_abort; ++u) {
        const int t = t0 + u / a.n_blocks, mb = u % a.n_blocks;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&empty[s], ((uint32_t)(it / S) & 1u) ^ 1u)) {
            *s_abort = 1;
            raise_flag(a.flags, DSPARK_FLAG_TIMEOUT);
            break;
          }
          uint8_t* st = ring + (size_t)s * kLhStage;
          mbar_arrive_expect_tx(&full[s], kLhStage);
          tma_load_2d_hint(st, &tm_h, &full[s], kb * 64, mb * 128, ph_);
          tma_load_2d(st + kStageBytes, &tm_e, &full[s], kb * 64, t * kTileN);
        }
      }
      // the MMAs' releases of the last stages (normal path), or the copies
      // still in flight (after an abort), before the CTA may exit
      if (!*s_abort) wait_ring_released(empty, S, it, a.flags);
      else drain_ring_loads(full, S, it);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, kTileN);
      const uint32_t r0 = smem_u32(ring);
      int it = 0;
      bool ok = true;
      for (int u = 0; u < n_units && ok && !*s_abort; ++u) {
        const int acc = u & 1;
        ok = mbar_wait(&accEmpty[acc], ((uint32_t)(u >> 1) & 1u) ^ 1u);
        if (!ok) break;
        tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          if (!(ok = mbar_wait(&full[s], (uint32_t)(it / S) & 1u))) break;
          tc_fence_after();
          const uint32_t sa = r0 + s * kLhStage, sb = sa + kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + acc * kTileN, sdesc_sw128(sa + kk * 32), sdesc_sw128(sb + kk * 32),
                        idesc, (kb | kk) != 0);
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&accFull[acc]);
      }
      if (!ok) {
        *s_abort = 1;
        raise_flag(a.flags, DSPARK_FLAG_TIMEOUT);
      }
      drain_mma(mmaDrain);
    }
  } else {
    // ---------------- epilogue: thread m = row m of the block (TMEM lane)
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;
    if (kMode == kLhStats) {
      for (int mb = 0; mb < a.n_blocks; ++mb)
        spart[mb * 128 + m] = make_float2(-CUDART_INF_F, 0.0f);
    }
    for (int u = 0; u < n_units; ++u) {
      const int t = t0 + u / a.n_blocks, mb = u % a.n_blocks;
      const int acc = u & 1;
      if (*s_abort || !mbar_wait(&accFull[acc], (uint32_t)(u >> 1) & 1u)) {
        *s_abort = 1;
        raise_flag(a.flags, DSPARK_FLAG_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int lr = mb * 128 + m;  // row of this launch
      const bool valid = lr < a.n_rows;
      int b = -1, x = -1;
      float it2 = kLog2e;
      if (kMode == kLhStats && valid) {
        const long long hr = a.row0 + lr;
        b = a.row_req[hr];
        if (b >= 0) {
          const int p = a.row_pos[hr];
          it2 = checked_inv_temp(a.inv_temp, b, a.flags) * kLog2e;
          const int L = a.verify_len[b];
          if (p < L) x = a.tokens[(size_t)b * a.K + p];  // ids were checked by the map
        }
      }
      float Mr = 0.0f, Sr = 0.0f;
      if (kMode == kLhStats && b >= 0) {
        const float2 q = spart[mb * 128 + m];
        Mr = q.x;
        Sr = q.y;
      }
#pragma unroll 1
      for (int cb = 0; cb < kTileN / 32; ++cb) {
        float d[32];
        tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + acc * kTileN + cb * 32, d);
        const int v0 = t * kTileN + cb * 32;
        if (kMode == kLhLogits) {
          if (valid) {
            float* dst = a.logits + (size_t)lr * a.V + v0;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              if (v0 + j < a.V)
                *reinterpret_cast<float4*>(dst + j) = make_float4(d[j], d[j + 1], d[j + 2], d[j + 3]);
          }
        } else if (b >= 0) {
          if (v0 + 32 > a.V) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (v0 + j >= a.V) d[j] = -CUDART_INF_F;
          }
          if (x >= v0 && x < v0 + 32) {
            float tx = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (v0 + j == x) tx = d[j];
            a.tok_logit[a.row0 + lr] = tx;
          }
          float A4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
          for (int j = 0; j < 32; ++j) A4[j & 3] = fmaxf(A4[j & 3], d[j]);
          const float A = fmaxf(fmaxf(A4[0], A4[1]), fmaxf(A4[2], A4[3]));
          if (A != -CUDART_INF_F) {
            float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int j = 0; j < 32; ++j) s4[j & 3] += ex2((d[j] - A) * it2);
            merge_partial(Mr, Sr, A, (s4[0] + s4[1]) + (s4[2] + s4[3]), it2);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accEmpty[acc]);
      if (kMode == kLhStats && b >= 0) spart[mb * 128 + m] = make_float2(Mr, Sr);
    }
    if (kMode == kLhStats && !*s_abort) {
      // this CTA's partial of every verified row of the launch
      for (int mb = 0; mb < a.n_blocks; ++mb) {
        const int lr = mb * 128 + m;
        if (lr >= a.n_rows) break;
        const long long hr = a.row0 + lr;
        const int b = a.row_req[hr];
        if (b < 0) continue;
        const int p = a.row_pos[hr];
        a.tpart[((size_t)b * (a.K + 1) + p) * G + g] = spart[mb * 128 + m];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kLhTmemCols);
}

// Map of the verified rows: row_req[row] = b, row_pos[row] = p for every
// (b, p <= L_b), row = row_start[b] + p (clamped like the verify's rows).
// A row claimed twice raises DSPARK_FLAG_BAD_LENGTH (the rows of the
// flattened verify are disjoint).  row_req must be -1 everywhere before.
__global__ void lm_row_map_kernel(const int64_t* __restrict__ row_start,
                                  const int32_t* __restrict__ verify_len,
                                  const int32_t* __restrict__ tokens, int V, int B, int K,
                                  long long n_rows, int* row_req, int* row_pos, unsigned* flags) {
  const int b = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  int L = verify_len[b];
  if (L < 0 || L > K) L = L < 0 ? 0 : K;  // the accept kernel raises the flag
  for (int p = lane; p <= L; p += 32) {
    long long row = (long long)row_start[b] + p;
    if (row < 0 || row >= n_rows) row = row < 0 ? 0 : n_rows - 1;  // flagged by the accept
    if (atomicCAS(&row_req[row], -1, b) != -1) {
      raise_flag(flags, DSPARK_FLAG_BAD_LENGTH);
    } else {
      row_pos[row] = p;
    }
    if (p < L) {
      const int x = tokens[(size_t)b * K + p];
      if (x < 0 || x >= V) raise_flag(flags, DSPARK_FLAG_BAD_TOKEN);
    }
  }
}

// The hidden row of every request's correction / bonus position, copied to
// a contiguous [B, dm] block (the A operand of the logits launch); the
// request's ResInfo then names its row of the scratch logits.
__global__ void lm_gather_rows_kernel(const __nv_bfloat16* __restrict__ hidden, int dm,
                                      ResInfo* info, __nv_bfloat16* __restrict__ rows, int B) {
  const int b = blockIdx.x;
  if (b >= B) return;
  const long long src = info[b].row;
  const uint4* s = reinterpret_cast<const uint4*>(hidden + (size_t)src * dm);
  uint4* d = reinterpret_cast<uint4*>(rows + (size_t)b * dm);
  for (int i = threadIdx.x; i < dm / 8; i += blockDim.x) d[i] = s[i];
  __syncthreads();
  if (threadIdx.x == 0) info[b].row = b;
}

// H [rows, dm] or E [V, dm] bf16 as 64 x 128 boxes, 128-byte swizzle.
inline bool encode_lh_map(CUtensorMap* m, const void* p, long long rows, int dm) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)dm, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)dm * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int lh_grid(int V) {
  const int n_tiles = (V + kTileN - 1) / kTileN;
  int G = num_sms();
  if (G > n_tiles) G = n_tiles;
  return G;
}

template <int kMode>
inline dspark_status lh_launch(const CUtensorMap& tm_h, const CUtensorMap& tm_e, LhArgs a,
                               cudaStream_t s) {
  static DeviceOnce once;
  set_smem_once(once, lmhead_tc_kernel<kMode>, (int)lh_smem_bytes());
  lmhead_tc_kernel<kMode><<<lh_grid(a.V), kLhThreads, lh_smem_bytes(), s>>>(tm_h, tm_e, a);
  return cudaGetLastError() == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

}  // namespace dspark
