// api.cu -- the C ABI (include/dspark.h): argument validation, workspace
// layout and kernel launches.  No entry point allocates memory or
// synchronises the stream (except the status readers).
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "prefix.cuh"
#include "proj_simt.cuh"
#include "proj_tc.cuh"
#include "draft_persist.cuh"
#include "sample.cuh"
#include "verify.cuh"
#include "verify_fused.cuh"
#include "sts.cuh"
#include "lmhead.cuh"
#include "rnn.cuh"

using namespace dspark;

namespace {

constexpr int kMaxK = 64;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Workspace of the draft: header (status word at 0, eight grid-barrier
// counters 128 bytes apart from byte 128), chunk partials [B][n_chunks],
// per-CTA partials [B][<=1024] (persistent paths: one per CTA; tensor-core
// path: one per CTA of the request's block and epilogue warpgroup), then
// (persistent paths) bias rows [B][V] and exchange records.
constexpr size_t kCounterOff = 128;
static_assert(kTcMaxCtasPerBlock * kS2Parts <= 1024, "per-CTA partials per request");
struct DraftWs {
  size_t part_off, cta_off, bias_off, rec_off, total;
};
DraftWs draft_ws(int V, int B) {
  DraftWs w;
  const int Bp = B <= kPMaxB ? B : 0;  // persistent paths only
  w.part_off = kHeaderBytes;
  w.cta_off = w.part_off + align256((size_t)B * n_chunks_of(V) * sizeof(float2));
  w.bias_off = w.cta_off + align256((size_t)B * 1024 * sizeof(float2));
  w.rec_off = w.bias_off + align256((size_t)Bp * V * sizeof(float));
  w.total = w.rec_off + align256(Bp ? gemv_rec_bytes(Bp) : 0);
  return w;
}

// Workspace of the verify: header, target partials [B*(K+1)][n_segs],
// ResInfo [B], residual partials [B][n_chunks], and (sizes the tensor-core
// path serves) the correction rows' bias [B][V].
struct VerifyWs {
  size_t frec_off, frec_bytes, tpart_off, info_off, rpart_off, total;
};
// Header, then the records of the fused small-batch verify (cleared together
// with the header, one memset), then the buffers of the multi-kernel path.
VerifyWs verify_ws(int V, int r, int B, int K) {
  VerifyWs w;
  w.frec_off = kHeaderBytes;
  w.frec_bytes = fused_verify_ok(B, K, true) ? align256(fused_rec_bytes(B)) : 0;
  w.tpart_off = w.frec_off + w.frec_bytes;
  w.info_off = w.tpart_off + align256((size_t)B * (K + 1) * n_segs_of(V) * sizeof(float2));
  w.rpart_off = w.info_off + align256((size_t)B * sizeof(ResInfo));
  w.total = w.rpart_off + align256((size_t)B * n_chunks_of(V) * sizeof(float2));
  return w;
}

dspark_status check_launch() {
  return cudaGetLastError() == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

// Clears the status word and the grid-barrier counters of a workspace.
dspark_status clear_status(void* ws, cudaStream_t s) {
  return cudaMemsetAsync(ws, 0, kHeaderBytes, s) == cudaSuccess ? DSPARK_OK : DSPARK_ERR_CUDA;
}

// Shape checks shared by draft and verify.
dspark_status check_shapes(int V, int r, int B, int K, dspark_dtype dt) {
  if (V <= 0 || r <= 0 || B < 0 || K < 0) return DSPARK_ERR_INVALID_ARG;
  if (dt != DSPARK_F32 && dt != DSPARK_BF16) return DSPARK_ERR_INVALID_ARG;
  if (V % 4 != 0 || r % 8 != 0) return DSPARK_ERR_UNSUPPORTED;
  if (r > kMaxRank || K > kMaxK) return DSPARK_ERR_UNSUPPORTED;
  if ((long long)V * (K + 1) > (1ll << 40)) return DSPARK_ERR_UNSUPPORTED;
  return DSPARK_OK;
}

int simt_group(int B) {
  int nb = 1;
  while (nb < B && nb < 16) nb <<= 1;
  return nb;
}

template <typename TW, int NB>
void launch_draft_proj_simt(const float* base, const void* U, const void* W, int V, int r, int B,
                            int K, int k, const int32_t* prev, const int32_t* tokens,
                            const float* it, float* dl, float* dbias, float2* part,
                            unsigned* flags, cudaStream_t s) {
  const int nc = n_chunks_of(V);
  const size_t smem = (size_t)NB * r * sizeof(float);
  static DeviceOnce once;
  set_smem_once(once, draft_proj_simt_kernel<TW, NB>, NB * kMaxRank * 4);
  dim3 grid((nc + 7) / 8, (B + NB - 1) / NB);
  draft_proj_simt_kernel<TW, NB><<<grid, 256, smem, s>>>(
      base, static_cast<const TW*>(U), static_cast<const TW*>(W), V, r, B, K, k, prev, tokens, it,
      dl, dbias, part, nc, flags);
}

template <typename TW, int NB>
void launch_res_proj_simt(const float* target, const float* base, const void* U, const void* W,
                          int V, int r, int B, int K, const ResInfo* info, const float* it,
                          float2* rpart, unsigned* flags, cudaStream_t s) {
  const int nc = n_chunks_of(V);
  const size_t smem = (size_t)NB * r * sizeof(float);
  static DeviceOnce once;
  set_smem_once(once, residual_proj_simt_kernel<TW, NB>, NB * kMaxRank * 4);
  dim3 grid((nc + 7) / 8, (B + NB - 1) / NB);
  residual_proj_simt_kernel<TW, NB><<<grid, 256, smem, s>>>(
      target, base, static_cast<const TW*>(U), static_cast<const TW*>(W), V, r, B, K, info, it,
      rpart, nc, flags);
}

template <typename TW>
void draft_proj_simt(int nb, const float* base, const void* U, const void* W, int V, int r, int B,
                     int K, int k, const int32_t* prev, const int32_t* tokens, const float* it,
                     float* dl, float* dbias, float2* part, unsigned* flags, cudaStream_t s) {
  switch (nb) {
    case 1: launch_draft_proj_simt<TW, 1>(base, U, W, V, r, B, K, k, prev, tokens, it, dl, dbias, part, flags, s); break;
    case 2: launch_draft_proj_simt<TW, 2>(base, U, W, V, r, B, K, k, prev, tokens, it, dl, dbias, part, flags, s); break;
    case 4: launch_draft_proj_simt<TW, 4>(base, U, W, V, r, B, K, k, prev, tokens, it, dl, dbias, part, flags, s); break;
    case 8: launch_draft_proj_simt<TW, 8>(base, U, W, V, r, B, K, k, prev, tokens, it, dl, dbias, part, flags, s); break;
    default: launch_draft_proj_simt<TW, 16>(base, U, W, V, r, B, K, k, prev, tokens, it, dl, dbias, part, flags, s); break;
  }
}

template <typename TW>
void res_proj_simt(int nb, const float* target, const float* base, const void* U, const void* W,
                   int V, int r, int B, int K, const ResInfo* info, const float* it, float2* rpart,
                   unsigned* flags, cudaStream_t s) {
  switch (nb) {
    case 1: launch_res_proj_simt<TW, 1>(target, base, U, W, V, r, B, K, info, it, rpart, flags, s); break;
    case 2: launch_res_proj_simt<TW, 2>(target, base, U, W, V, r, B, K, info, it, rpart, flags, s); break;
    case 4: launch_res_proj_simt<TW, 4>(target, base, U, W, V, r, B, K, info, it, rpart, flags, s); break;
    case 8: launch_res_proj_simt<TW, 8>(target, base, U, W, V, r, B, K, info, it, rpart, flags, s); break;
    default: launch_res_proj_simt<TW, 16>(target, base, U, W, V, r, B, K, info, it, rpart, flags, s); break;
  }
}

// Which projection path a draft / residual of these sizes takes.
bool use_tc(int V, int r, int B, dspark_dtype dt) {
  return dt == DSPARK_BF16 && B > 16 && tc_supported(V, r, B);
}
bool use_persist(int V, int r, int B, dspark_dtype dt) {
  return dt == DSPARK_BF16 && persist_supported(V, r, B);
}

template <typename TW>
dspark_status draft_impl(const float* base, const void* U, const void* W, dspark_dtype dt, int V,
                         int r, int B, int K, const int32_t* prev, const float* it,
                         const float* ud, int32_t* tokens, float* p_tok, float* lse, float* rmax,
                         float* rsum, float* dl, float* dbias, unsigned char* ws, cudaStream_t s) {
  const DraftWs w = draft_ws(V, B);
  unsigned* flags = reinterpret_cast<unsigned*>(ws);
  float2* part = reinterpret_cast<float2*>(ws + w.part_off);
  const int nc = n_chunks_of(V);
  if (use_persist(V, r, B, dt)) {
    CUtensorMap tm_w;
    if (!encode_w_map(&tm_w, W, V, r)) return DSPARK_ERR_CUDA;
    PersistArgs a;
    a.base = base;
    a.U = static_cast<const __nv_bfloat16*>(U);
    a.W = static_cast<const __nv_bfloat16*>(W);
    a.prev_token = prev;
    a.inv_temp = it;
    a.u_draft = ud;
    a.tokens = tokens;
    a.p_tok = p_tok;
    a.lse = lse;
    a.ref_max = rmax;
    a.ref_sum = rsum;
    a.draft_logits = dl;
    a.part = part;
    a.cta_part = reinterpret_cast<float2*>(ws + w.cta_off);
    a.bias_buf = reinterpret_cast<float*>(ws + w.bias_off);
    a.draft_bias = dbias;
    a.flags = flags;
    a.grid_counter = reinterpret_cast<unsigned*>(ws + kCounterOff);
    a.V = V;
    a.r = r;
    a.B = B;
    a.K = K;
    a.n_chunks = nc;
    a.n_tiles = (V + kTileN - 1) / kTileN;
    GemvRecs recs;
    recs.cta = reinterpret_cast<unsigned long long*>(ws + w.rec_off);
    recs.tok = recs.cta + gemv_rec_words_cta(B);
    if (gemv_path(r, B) &&
        cudaMemsetAsync(ws + w.rec_off, 0, gemv_rec_bytes(B), s) != cudaSuccess)
      return DSPARK_ERR_CUDA;
    dspark_status st = persist_launch(tm_w, a, recs, s);
    if (st != DSPARK_OK) return st;
    return check_launch();
  }
  const bool tc = use_tc(V, r, B, dt);
  TcPlan plan;
  if (tc) {
    dspark_status st = tc_plan_draft(plan, base, U, W, V, r, B, K);
    if (st != DSPARK_OK) return st;
  }
  const int nb = simt_group(B);
  float2* cta_part = reinterpret_cast<float2*>(ws + w.cta_off);
  for (int k = 0; k < K; ++k) {
    if (tc) {
      tc_launch_draft(plan, k, prev, tokens, it, dl, dbias, part, cta_part, flags, s);
      // two-level sampler over the projection's CTA partials, a warp per request
      draft_sample2_kernel<TW><<<(B + kS2Warps - 1) / kS2Warps, kS2Warps * 32, 0, s>>>(
          base, static_cast<const TW*>(U), static_cast<const TW*>(W), V, r, B, K, k, prev,
          tokens, it, ud, part, nc, cta_part, plan.ctas_per_bb, plan.n_tiles, dbias, p_tok, lse,
          rmax, rsum, flags);
    } else {
      draft_proj_simt<TW>(nb, base, U, W, V, r, B, K, k, prev, tokens, it, dl, dbias, part, flags, s);
      draft_sample_kernel<TW><<<B, kSampleThreads, 0, s>>>(
          base, static_cast<const TW*>(U), static_cast<const TW*>(W), V, r, K, k, prev, tokens,
          it, ud, part, nc, dbias, p_tok, lse, rmax, rsum, flags);
    }
  }
  return check_launch();
}

// The verify's last two stages, shared by the stored-logits and the LM-head
// verify: residual partials of every request's correction / bonus row (from
// the draft's bias rows, or re-projected on the tensor or CUDA cores), then
// the draw.  `target` holds that row of request b at info[b].row.
// With the tensor cores (large batches, no bias rows from the draft) one
// projection re-forms the correction rows' bias and reduces the residual in
// its epilogue, the per-request target and base row segments fetched by TMA
// gathers.  (Projecting the bias rows to a [B, V] buffer first and then
// streaming target, base and bias rows measured 0.89 against 0.70 ms at
// B = 512, V = 151936.)
template <typename TW>
dspark_status residual_tail(const float* target, long long n_rows, const float* base,
                            const void* U, const void* W, dspark_dtype dt, int V, int r, int B,
                            int K, const float* it, const float* ur, const ResInfo* info,
                            float2* rpart, const float* dbias, int32_t* out,
                            int32_t* last, unsigned* flags, cudaStream_t s) {
  (void)n_rows;
  const int nc = n_chunks_of(V);
  dim3 rgrid((nc + 7) / 8, B);
  if (dbias != nullptr) {
    residual_bias_kernel<<<rgrid, 256, 0, s>>>(target, base, dbias, V, K, info, it, rpart, nc,
                                                flags);
  } else if (use_tc(V, r, B, dt)) {
    TcPlan plan;
    dspark_status st = tc_plan_residual(plan, target, n_rows, base, U, W, V, r, B, K);
    if (st != DSPARK_OK) return st;
    tc_launch_residual(plan, info, it, rpart, flags, s);
  } else {
    res_proj_simt<TW>(simt_group(B), target, base, U, W, V, r, B, K, info, it, rpart, flags, s);
  }
  residual_sample_kernel<TW><<<B, kSampleThreads, 0, s>>>(
      target, base, static_cast<const TW*>(U), static_cast<const TW*>(W), V, r, K, it, ur, info,
      rpart, nc, dbias, out, last, flags);
  return check_launch();
}

template <typename TW>
dspark_status verify_impl(const float* target, long long n_rows, const int64_t* row_start,
                          const int32_t* vlen, const float* base, const void* U, const void* W,
                          dspark_dtype dt, int V, int r, int B, int K, const int32_t* prev,
                          const float* it, const int32_t* tokens, const float* p_tok,
                          const float* rmax, const float* rsum, const float* dbias,
                          const float* ua, const float* ur, int32_t* n_acc, int32_t* out,
                          int32_t* last, unsigned char* ws, cudaStream_t s) {
  const VerifyWs w = verify_ws(V, r, B, K);
  unsigned* flags = reinterpret_cast<unsigned*>(ws);
  const int nc = n_chunks_of(V);
  const int G = fused_grid(V, B * (K + 1));
  if (dbias != nullptr && w.frec_bytes > 0 && G > 0) {
    // one cooperative launch; its records are cleared with the status word
    if (cudaMemsetAsync(ws, 0, kHeaderBytes + w.frec_bytes, s) != cudaSuccess) return DSPARK_ERR_CUDA;
    FusedArgs a;
    a.target = target;
    a.n_rows = n_rows;
    a.row_start = row_start;
    a.verify_len = vlen;
    a.base = base;
    a.draft_bias = dbias;
    a.inv_temp = it;
    a.prev_token = prev;
    a.tokens = tokens;
    a.p_tok = p_tok;
    a.ref_max = rmax;
    a.ref_sum = rsum;
    a.u_accept = ua;
    a.u_res = ur;
    a.n_accepted = n_acc;
    a.out_tokens = out;
    a.last_token = last;
    a.flags = flags;
    a.seg_rec = reinterpret_cast<unsigned long long*>(ws + w.frec_off);
    a.tot_rec = a.seg_rec + kFSegWords;
    a.V = V;
    a.B = B;
    a.K = K;
    a.n_chunks = nc;
    static DeviceOnce once;
    set_smem_once(once, verify_fused_kernel, kFBufFloats * (int)sizeof(float));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = kFBufFloats * sizeof(float);
    cfg.stream = s;
    cudaLaunchAttribute attrs[1];
    attrs[0].id = cudaLaunchAttributeCooperative;
    attrs[0].val.cooperative = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, verify_fused_kernel, a) != cudaSuccess) return DSPARK_ERR_CUDA;
    return check_launch();
  }
  dspark_status st0 = clear_status(ws, s);
  if (st0 != DSPARK_OK) return st0;
  float2* tpart = reinterpret_cast<float2*>(ws + w.tpart_off);
  ResInfo* info = reinterpret_cast<ResInfo*>(ws + w.info_off);
  float2* rpart = reinterpret_cast<float2*>(ws + w.rpart_off);
  const int ns = n_segs_of(V);
  dim3 sgrid(ns, B * (K + 1));
  target_stats_kernel<<<sgrid, kStatsThreads, 0, s>>>(target, n_rows, row_start, vlen, it, V, K,
                                                       tpart, ns, flags);
  accept_kernel<<<(B + 3) / 4, 128, 0, s>>>(target, n_rows, row_start, vlen, it, V, B, K, prev,
                                            tokens, p_tok, rmax, rsum, ua, tpart, ns, n_acc, out,
                                            info, flags);
  return residual_tail<TW>(target, n_rows, base, U, W, dt, V, r, B, K, it, ur, info, rpart, dbias,
                           out, last, flags, s);
}

// ---------------------------------------------------------------------------
// Verify with the target logits formed from hidden states and the LM head
// ---------------------------------------------------------------------------
// Workspace: header, the row map (request and position of every hidden row),
// the drafted tokens' raw logits, per-CTA partials of every verified row,
// ResInfo, the correction rows' hidden states [B, dm] and logits [B, V], the
// residual partials.
constexpr int kLhMaxG = 256;
constexpr int kLhMaxDm = 16384;
struct LmWs {
  size_t map_off, pos_off, tok_off, tpart_off, info_off, rows_off, logits_off, rpart_off, total;
};
LmWs lm_ws(int V, int r, int B, int K, int dm, long long n_rows) {
  LmWs w;
  w.map_off = kHeaderBytes;
  w.pos_off = w.map_off + align256((size_t)n_rows * 4);
  w.tok_off = w.pos_off + align256((size_t)n_rows * 4);
  w.tpart_off = w.tok_off + align256((size_t)n_rows * 4);
  w.info_off = w.tpart_off + align256((size_t)B * (K + 1) * kLhMaxG * sizeof(float2));
  w.rows_off = w.info_off + align256((size_t)B * sizeof(ResInfo));
  w.logits_off = w.rows_off + align256((size_t)B * dm * 2);
  w.rpart_off = w.logits_off + align256((size_t)B * V * 4);
  w.total = w.rpart_off + align256((size_t)B * n_chunks_of(V) * sizeof(float2));
  return w;
}

template <typename TW>
dspark_status verify_lmhead_impl(const void* hidden, const void* head, int dm, long long n_rows,
                                 const int64_t* row_start, const int32_t* vlen, const float* base,
                                 const void* U, const void* W, dspark_dtype dt, int V, int r,
                                 int B, int K, const int32_t* prev, const float* it,
                                 const int32_t* tokens, const float* p_tok, const float* rmax,
                                 const float* rsum, const float* dbias, const float* ua,
                                 const float* ur, int32_t* n_acc, int32_t* out, int32_t* last,
                                 unsigned char* ws, cudaStream_t s) {
  const LmWs w = lm_ws(V, r, B, K, dm, n_rows);
  unsigned* flags = reinterpret_cast<unsigned*>(ws);
  int* row_req = reinterpret_cast<int*>(ws + w.map_off);
  int* row_pos = reinterpret_cast<int*>(ws + w.pos_off);
  float* tok_logit = reinterpret_cast<float*>(ws + w.tok_off);
  float2* tpart = reinterpret_cast<float2*>(ws + w.tpart_off);
  ResInfo* info = reinterpret_cast<ResInfo*>(ws + w.info_off);
  __nv_bfloat16* rows = reinterpret_cast<__nv_bfloat16*>(ws + w.rows_off);
  float* logits = reinterpret_cast<float*>(ws + w.logits_off);
  float2* rpart = reinterpret_cast<float2*>(ws + w.rpart_off);
  const int G = lh_grid(V);
  if (G > kLhMaxG) return DSPARK_ERR_UNSUPPORTED;
  dspark_status st = clear_status(ws, s);
  if (st != DSPARK_OK) return st;
  if (cudaMemsetAsync(row_req, 0xFF, (size_t)n_rows * 4, s) != cudaSuccess) return DSPARK_ERR_CUDA;
  lm_row_map_kernel<<<(B + 3) / 4, 128, 0, s>>>(row_start, vlen, tokens, V, B, K, n_rows, row_req,
                                                row_pos, flags);
  CUtensorMap tm_e;
  if (!encode_lh_map(&tm_e, head, V, dm)) return DSPARK_ERR_CUDA;
  const __nv_bfloat16* H = static_cast<const __nv_bfloat16*>(hidden);
  LhArgs a = {};
  a.dm = dm;
  a.V = V;
  a.n_tiles = (V + kTileN - 1) / kTileN;
  a.row_req = row_req;
  a.row_pos = row_pos;
  a.inv_temp = it;
  a.tokens = tokens;
  a.verify_len = vlen;
  a.K = K;
  a.tpart = tpart;
  a.tok_logit = tok_logit;
  a.flags = flags;
  // 1. softmax partials of every verified row (and the drafted tokens'
  //    logits), up to 2048 hidden rows per launch
  constexpr long long kRowsPerLaunch = (long long)kLhMaxBlocks * 128;
  for (long long r0 = 0; r0 < n_rows; r0 += kRowsPerLaunch) {
    const long long nr = n_rows - r0 < kRowsPerLaunch ? n_rows - r0 : kRowsPerLaunch;
    CUtensorMap tm_h;
    if (!encode_lh_map(&tm_h, H + (size_t)r0 * dm, nr, dm)) return DSPARK_ERR_CUDA;
    a.n_rows = (int)nr;
    a.row0 = r0;
    a.n_blocks = (int)((nr + 127) / 128);
    if ((st = lh_launch<kLhStats>(tm_h, tm_e, a, s)) != DSPARK_OK) return st;
  }
  // 2. accept scan on those partials
  accept_kernel<<<(B + 3) / 4, 128, 0, s>>>(nullptr, n_rows, row_start, vlen, it, V, B, K, prev,
                                            tokens, p_tok, rmax, rsum, ua, tpart, G, n_acc, out,
                                            info, flags, tok_logit);
  // 3. the logits of every request's correction / bonus row, to scratch
  lm_gather_rows_kernel<<<B, 128, 0, s>>>(H, dm, info, rows, B);
  for (long long r0 = 0; r0 < B; r0 += kRowsPerLaunch) {
    const long long nr = B - r0 < kRowsPerLaunch ? B - r0 : kRowsPerLaunch;
    CUtensorMap tm_h;
    if (!encode_lh_map(&tm_h, rows + (size_t)r0 * dm, nr, dm)) return DSPARK_ERR_CUDA;
    a.n_rows = (int)nr;
    a.row0 = 0;
    a.n_blocks = (int)((nr + 127) / 128);
    a.logits = logits + (size_t)r0 * V;
    if ((st = lh_launch<kLhLogits>(tm_h, tm_e, a, s)) != DSPARK_OK) return st;
  }
  // 4. residual and draw, as in the stored-logits verify
  return residual_tail<TW>(logits, B, base, U, W, dt, V, r, B, K, it, ur, info, rpart, dbias,
                           out, last, flags, s);
}

// ---------------------------------------------------------------------------
// Verify without a caller-provided workspace
// ---------------------------------------------------------------------------
// Scratch of dspark_verify_noalloc: a fixed array in the library image, so a
// caller that cannot allocate device memory can still run the verify.  Every
// GPU that loads the library holds these bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;  // 2 MiB
static __device__ __align__(256) unsigned char g_verify_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch on the current device.  Host code may not
// use the symbol itself (it names a host-side stand-in); the address comes
// from cudaGetSymbolAddress, looked up once per device with that device
// current and cached.
dspark_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSPARK_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return DSPARK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_verify_scratch) != cudaSuccess || p == nullptr)
      return DSPARK_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DSPARK_OK;
}

}  // namespace

extern "C" {

int dspark_version(void) { return 101; }

const char* dspark_status_string(dspark_status s) {
  switch (s) {
    case DSPARK_OK: return "ok";
    case DSPARK_ERR_INVALID_ARG: return "invalid argument";
    case DSPARK_ERR_CUDA: return "CUDA runtime error";
    case DSPARK_ERR_TIMEOUT: return "device wait timed out";
    case DSPARK_ERR_UNSUPPORTED: return "sizes not supported by this library";
    case DSPARK_ERR_DEVICE_DATA: return "device found invalid data";
    case DSPARK_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

const char* dspark_draft_path(int V, int r, int B, int K, dspark_dtype uw_dtype) {
  (void)K;
  if (use_persist(V, r, B, uw_dtype))
    return gemv_path(r, B) ? "persistent-cuda-core" : "tcgen05-persistent";
  return use_tc(V, r, B, uw_dtype) ? "tcgen05" : "cuda-core";
}

const char* dspark_prefix_path(int B, int K, int enable) {
  if (B < 0 || K < 0) return "single-cta";
  return prefix_multi(B * K, enable) ? "multi-cta" : "single-cta";
}

const char* dspark_verify_path(int V, int r, int B, int K, dspark_dtype uw_dtype, int have_bias) {
  if (fused_verify_ok(B, K, have_bias != 0) && fused_grid(V, B * (K + 1)) > 0)
    return "single-launch";
  if (have_bias) return "staged-bias";
  return use_tc(V, r, B, uw_dtype) ? "staged-tcgen05" : "staged-cuda-core";
}

size_t dspark_draft_workspace_size(int V, int r, int B, int K) {
  (void)r;
  (void)K;
  if (V <= 0 || B < 0) return 0;
  return draft_ws(V, B).total;
}

size_t dspark_verify_workspace_size(int V, int r, int B, int K) {
  (void)r;
  if (V <= 0 || B < 0 || K < 0) return 0;
  return verify_ws(V, r, B, K).total;
}

size_t dspark_prefix_workspace_size(int B, int K, int n_pts) {
  (void)n_pts;
  if (B < 0 || K < 0 || (long long)B * K > kMaxCand) return kHeaderBytes;
  return prefix_ws_bytes(B * K);
}

dspark_status dspark_draft_markov(const float* base_logits, const void* U, const void* W,
                                  dspark_dtype uw_dtype, int V, int r, int B, int K,
                                  const int32_t* prev_token, const float* inv_temp,
                                  const float* u_draft, int32_t* tokens, float* p_tok, float* lse,
                                  float* ref_max, float* ref_sum, float* draft_logits,
                                  float* draft_bias, void* workspace, size_t ws_bytes,
                                  void* stream) {
  dspark_status st = check_shapes(V, r, B, K, uw_dtype);
  if (st != DSPARK_OK) return st;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < dspark_draft_workspace_size(V, r, B, K))
    return DSPARK_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 0 || K == 0) return clear_status(workspace, s);
  if (!base_logits || !U || !W || !prev_token || !u_draft || !tokens || !p_tok || !lse ||
      !ref_max || !ref_sum)
    return DSPARK_ERR_INVALID_ARG;
  if (!aligned(base_logits, 16) || !aligned(U, 16) || !aligned(W, 16) ||
      (draft_logits && !aligned(draft_logits, 16)) || (draft_bias && !aligned(draft_bias, 16)))
    return DSPARK_ERR_INVALID_ARG;
  if ((st = clear_status(workspace, s)) != DSPARK_OK) return st;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (uw_dtype == DSPARK_BF16)
    return draft_impl<__nv_bfloat16>(base_logits, U, W, uw_dtype, V, r, B, K, prev_token,
                                     inv_temp, u_draft, tokens, p_tok, lse, ref_max, ref_sum,
                                     draft_logits, draft_bias, ws, s);
  return draft_impl<float>(base_logits, U, W, uw_dtype, V, r, B, K, prev_token, inv_temp, u_draft,
                           tokens, p_tok, lse, ref_max, ref_sum, draft_logits, draft_bias, ws, s);
}

dspark_status dspark_verify(const float* target_logits, int64_t n_target_rows,
                            const int64_t* row_start, const int32_t* verify_len,
                            const float* base_logits, const void* U, const void* W,
                            dspark_dtype uw_dtype, int V, int r, int B, int K,
                            const int32_t* prev_token, const float* inv_temp,
                            const int32_t* tokens, const float* p_tok, const float* ref_max,
                            const float* ref_sum, const float* draft_bias, const float* u_accept,
                            const float* u_resample, int32_t* n_accepted, int32_t* out_tokens,
                            int32_t* last_token,
                            void* workspace, size_t ws_bytes, void* stream) {
  dspark_status st = check_shapes(V, r, B, K, uw_dtype);
  if (st != DSPARK_OK) return st;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < dspark_verify_workspace_size(V, r, B, K))
    return DSPARK_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 0) return clear_status(workspace, s);
  if (!target_logits || n_target_rows <= 0 || !row_start || !verify_len || !base_logits || !U ||
      !W || !prev_token || !u_resample || !n_accepted || !out_tokens)
    return DSPARK_ERR_INVALID_ARG;
  if (K > 0 && (!tokens || !p_tok || !ref_max || !ref_sum || !u_accept))
    return DSPARK_ERR_INVALID_ARG;
  if (!aligned(target_logits, 16) || !aligned(base_logits, 16) || !aligned(U, 16) ||
      !aligned(W, 16))
    return DSPARK_ERR_INVALID_ARG;
  if ((long long)B * (K + 1) > (1ll << 31) - 1) return DSPARK_ERR_UNSUPPORTED;
  // verify_impl clears the status word (and its records) before its kernels
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (uw_dtype == DSPARK_BF16)
    return verify_impl<__nv_bfloat16>(target_logits, n_target_rows, row_start, verify_len,
                                      base_logits, U, W, uw_dtype, V, r, B, K, prev_token,
                                      inv_temp, tokens, p_tok, ref_max, ref_sum, draft_bias,
                                      u_accept, u_resample, n_accepted, out_tokens, last_token, ws,
                                      s);
  return verify_impl<float>(target_logits, n_target_rows, row_start, verify_len, base_logits, U, W,
                            uw_dtype, V, r, B, K, prev_token, inv_temp, tokens, p_tok, ref_max,
                            ref_sum, draft_bias, u_accept, u_resample, n_accepted, out_tokens,
                            last_token, ws, s);
}

dspark_status dspark_confidence_prefix_async(const float* z, const float* temps,
                                             const float* cost_tokens, const float* cost_ms,
                                             int n_pts, int staircase, int B, int K, int enable,
                                             const int32_t* budget_in, float* c, float* survival,
                                             int32_t* verify_len, float* objective,
                                             int32_t* budget_out, void* workspace,
                                             size_t ws_bytes, void* stream) {
  if (B < 0 || K < 0 || n_pts < 2 || n_pts > 64 || (staircase != 0 && staircase != 1))
    return DSPARK_ERR_INVALID_ARG;
  if ((long long)B * K > kMaxCand) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < dspark_prefix_workspace_size(B, K, n_pts))
    return DSPARK_ERR_WORKSPACE;
  if (!cost_tokens || !cost_ms || !verify_len || !objective) return DSPARK_ERR_INVALID_ARG;
  if (B * K > 0 && (!z || !temps || !c || !survival)) return DSPARK_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = B * K;
  const PrefixArgs a{z, temps, cost_tokens, cost_ms, n_pts, staircase, B, K, enable,
                     budget_in, c, survival, verify_len, objective, budget_out,
                     static_cast<unsigned*>(workspace)};
  if (prefix_multi(n, enable)) {
    // survival pass, then the rank pass behind it (dependent launch); the
    // survival pass clears the status word and the rank counter
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    double* surv = reinterpret_cast<double*>(ws + kHeaderBytes);
    double* okey = reinterpret_cast<double*>(ws + kHeaderBytes + align256((size_t)n * 8));
    int* oidx = reinterpret_cast<int*>(ws + kHeaderBytes + 2 * align256((size_t)n * 8));
    unsigned* counter = reinterpret_cast<unsigned*>(ws + kPrefixCounterOff);
    static DeviceOnce once_multi;
    once_per_device(once_multi, [] {
      cudaFuncSetAttribute(prefix_surv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kMaxCand * (int)sizeof(double));
      cudaFuncSetAttribute(prefix_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kMaxCand * 16);
    });
    const int rb = K >= kSurvThreads ? 1 : kSurvThreads / K;
    prefix_surv_kernel<<<(B + rb - 1) / rb, kSurvThreads, (size_t)rb * K * sizeof(double), s>>>(
        a, surv, counter);
    dspark_status st = check_launch();
    if (st != DSPARK_OK) return st;
    // the last CTA's copy of the order and the per-request counts
    const size_t smem = (size_t)n * (sizeof(double) + sizeof(int)) + (size_t)B * sizeof(int);
    if (launch_dependent(prefix_rank_kernel, dim3((n + kRankSlice - 1) / kRankSlice),
                         dim3(kRankThreads), smem, s, a, static_cast<const double*>(surv), okey,
                         oidx, counter) != cudaSuccess)
      return DSPARK_ERR_CUDA;
    return check_launch();
  }
  // the merge's two buffers of (survival fp64, candidate id) and the
  // per-request counts
  const size_t smem = (size_t)n * 2 * (sizeof(double) + sizeof(int)) + (size_t)B * sizeof(int);
  constexpr int kPrefixSmemMax = kMaxCand * 24 + kMaxCand * 4;
  static DeviceOnce once;
  set_smem_once(once, prefix_kernel<kPrefixThreads>, kPrefixSmemMax);
  if (smem > (size_t)kPrefixSmemMax) return DSPARK_ERR_UNSUPPORTED;
  // the kernel clears the status word itself (one CTA: before any flag is raised)
  if (n <= kPrefixSmallCand)
    prefix_kernel<kPrefixThreadsSmall><<<1, kPrefixThreadsSmall, smem, s>>>(a);
  else
    prefix_kernel<kPrefixThreads><<<1, kPrefixThreads, smem, s>>>(a);
  return check_launch();
}

dspark_status dspark_confidence_prefix(const float* z, const float* temps,
                                       const float* cost_tokens, const float* cost_ms, int n_pts,
                                       int B, int K, int enable, float* c, float* survival,
                                       int32_t* verify_len, float* objective, void* workspace,
                                       size_t ws_bytes, void* stream) {
  return dspark_confidence_prefix_async(z, temps, cost_tokens, cost_ms, n_pts, 0, B, K, enable,
                                        nullptr, c, survival, verify_len, objective, nullptr,
                                        workspace, ws_bytes, stream);
}

// Workspace of the temperature fit: header, search state per position and
// the active count, derivative partials [G][K][4], calibration-error
// partials [G][31].
struct StsWs {
  size_t pos_off, part_off, bpart_off, total;
};
StsWs sts_ws(long long N, int K) {
  const int G = sts_grid(N);
  StsWs w;
  w.pos_off = kHeaderBytes;
  w.part_off = w.pos_off + align256(kStsPosBytes);
  w.bpart_off = w.part_off + align256((size_t)G * K * kStsPart * sizeof(double));
  w.total = w.bpart_off + align256((size_t)G * kStsBinVals * sizeof(double));
  return w;
}

size_t dspark_sts_workspace_size(long long N, int K) {
  if (N < 0 || K < 1 || K > kStsMaxK) return 0;
  return sts_ws(N, K).total;
}

dspark_status dspark_sts_fit(const float* z, const int32_t* n_accepted, long long N, int K,
                             float* temps, float* ece, int32_t* passes, void* workspace,
                             size_t ws_bytes, void* stream) {
  if (N < 0 || K < 1) return DSPARK_ERR_INVALID_ARG;
  if (K > kStsMaxK) return DSPARK_ERR_UNSUPPORTED;
  if (!temps || !ece || (N > 0 && (!z || !n_accepted))) return DSPARK_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < sts_ws(N, K).total)
    return DSPARK_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dspark_status st = clear_status(workspace, s);
  if (st != DSPARK_OK) return st;
  const StsWs w = sts_ws(N, K);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  unsigned* flags = reinterpret_cast<unsigned*>(ws);
  StsPos* pos = reinterpret_cast<StsPos*>(ws + w.pos_off);
  int* n_active = reinterpret_cast<int*>(ws + w.pos_off + sizeof(StsPos) * kStsMaxK);
  double* part = reinterpret_cast<double*>(ws + w.part_off);
  double* bpart = reinterpret_cast<double*>(ws + w.bpart_off);
  const int G = sts_grid(N);
  sts_init_kernel<<<1, 32, 0, s>>>(pos, n_active, K);
  // bounds at steps 0 and 1, then Newton steps; a pass with nothing left to
  // search returns at once
  const int last = 1 + kStsIters;
  for (int step = 0; step <= last; ++step) {
    if (step == 0)
      sts_grad_kernel<true><<<G, kStsThreads, 0, s>>>(z, n_accepted, N, K, pos, n_active, part,
                                                       flags);
    else
      sts_grad_kernel<false><<<G, kStsThreads, 0, s>>>(z, n_accepted, N, K, pos, n_active, part,
                                                        flags);
    sts_update_kernel<<<1, 32 * K, 0, s>>>(part, G, K, pos, n_active, step, last, temps, passes);
  }
  for (int fitted = 0; fitted < 2; ++fitted) {
    sts_ece_kernel<<<G, kStsThreads, 0, s>>>(z, n_accepted, N, K, pos, !fitted, bpart, flags);
    sts_ece_final_kernel<<<1, 32 * kStsBinVals, 0, s>>>(bpart, G, ece + fitted);
  }
  return check_launch();
}

int dspark_get_device_flags(const void* workspace, void* stream) {
  if (!workspace) return -1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned h = 0;
  if (cudaMemcpyAsync(&h, workspace, sizeof h, cudaMemcpyDeviceToHost, s) != cudaSuccess) return -1;
  if (cudaStreamSynchronize(s) != cudaSuccess) return -1;
  return (int)(h & 0x7fffffffu);  // -1 stays reserved for CUDA errors
}

dspark_status dspark_get_device_status(const void* workspace, void* stream) {
  const int f = dspark_get_device_flags(workspace, stream);
  if (f < 0) return DSPARK_ERR_CUDA;
  if (f & DSPARK_FLAG_TIMEOUT) return DSPARK_ERR_TIMEOUT;
  if (f) return DSPARK_ERR_DEVICE_DATA;
  return DSPARK_OK;
}

dspark_status dspark_verify_noalloc(const float* target_logits, int64_t n_target_rows,
                                    const int64_t* row_start, const int32_t* verify_len,
                                    const float* base_logits, const void* U, const void* W,
                                    dspark_dtype uw_dtype, int V, int r, int B, int K,
                                    const int32_t* prev_token, const float* inv_temp,
                                    const int32_t* tokens, const float* p_tok,
                                    const float* ref_max, const float* ref_sum,
                                    const float* draft_bias, const float* u_accept,
                                    const float* u_resample, int32_t* n_accepted,
                                    int32_t* out_tokens, int32_t* last_token, void* stream) {
  // sizes first: nothing below runs for a problem that does not fit
  const dspark_status st0 = check_shapes(V, r, B, K, uw_dtype);
  if (st0 != DSPARK_OK) return st0;
  if (dspark_verify_workspace_size(V, r, B, K) > kNoAllocScratchBytes) return DSPARK_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const dspark_status st = noalloc_scratch(&scratch);
  if (st != DSPARK_OK) return st;
  return dspark_verify(target_logits, n_target_rows, row_start, verify_len, base_logits, U, W,
                       uw_dtype, V, r, B, K, prev_token, inv_temp, tokens, p_tok, ref_max, ref_sum,
                       draft_bias, u_accept, u_resample, n_accepted, out_tokens, last_token, scratch,
                       kNoAllocScratchBytes, stream);
}

size_t dspark_draft_rnn_workspace_size(int V, int r, int B, int K) {
  (void)K;
  if (V <= 0 || r <= 0 || B < 0) return 0;
  return draft_ws(V, B).total + align256((size_t)B * r * 4) + align256((size_t)B * 2 * r * 2);
}

dspark_status dspark_draft_rnn(const float* base_logits, const void* U, const void* W,
                               const void* R, dspark_dtype uw_dtype, int V, int r, int B, int K,
                               const int32_t* prev_token, const float* h0, const float* inv_temp,
                               const float* u_draft, int32_t* tokens, float* p_tok, float* lse,
                               float* ref_max, float* ref_sum, float* states,
                               float* draft_logits, float* draft_bias, void* workspace,
                               size_t ws_bytes, void* stream) {
  dspark_status st = check_shapes(V, r, B, K, uw_dtype);
  if (st != DSPARK_OK) return st;
  // the state's projection runs on the tensor cores: bf16 factors, r a
  // multiple of 64 up to 256, one full vocabulary tile at least
  if (uw_dtype != DSPARK_BF16 || r % 64 != 0 || r > 256 || V < kTileN)
    return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || !aligned(workspace, 256) ||
      ws_bytes < dspark_draft_rnn_workspace_size(V, r, B, K))
    return DSPARK_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 0 || K == 0) return clear_status(workspace, s);
  if (!base_logits || !U || !W || !R || !prev_token || !u_draft || !tokens || !p_tok || !lse ||
      !ref_max || !ref_sum)
    return DSPARK_ERR_INVALID_ARG;
  if (!aligned(base_logits, 16) || !aligned(U, 16) || !aligned(W, 16) || !aligned(R, 16) ||
      (draft_logits && !aligned(draft_logits, 16)) || (draft_bias && !aligned(draft_bias, 16)))
    return DSPARK_ERR_INVALID_ARG;
  if ((st = clear_status(workspace, s)) != DSPARK_OK) return st;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  const DraftWs w = draft_ws(V, B);
  unsigned* flags = reinterpret_cast<unsigned*>(ws);
  float2* part = reinterpret_cast<float2*>(ws + w.part_off);
  float2* cta_part = reinterpret_cast<float2*>(ws + w.cta_off);
  float* state = reinterpret_cast<float*>(ws + w.total);
  __nv_bfloat16* a_rows =
      reinterpret_cast<__nv_bfloat16*>(ws + w.total + align256((size_t)B * r * 4));
  TcPlan plan;
  if ((st = tc_plan_draft(plan, base_logits, U, W, V, r, B, K, a_rows)) != DSPARK_OK) return st;
  const __nv_bfloat16* Ub = static_cast<const __nv_bfloat16*>(U);
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(W);
  const __nv_bfloat16* Rb = static_cast<const __nv_bfloat16*>(R);
  const int nc = n_chunks_of(V);
  for (int k = 0; k < K; ++k) {
    // state, then the projection of the state, then the draw
    rnn_state_kernel<__nv_bfloat16><<<B, kRnnThreads, (size_t)r * sizeof(float), s>>>(
        Ub, Rb, V, r, K, k, prev_token, tokens, h0, state, a_rows, states, flags);
    tc_launch_draft(plan, k, prev_token, tokens, inv_temp, draft_logits, draft_bias, part,
                    cta_part, flags, s);
    draft_sample2_kernel<__nv_bfloat16><<<(B + kS2Warps - 1) / kS2Warps, kS2Warps * 32, 0, s>>>(
        base_logits, Ub, Wb, V, r, B, K, k, prev_token, tokens, inv_temp, u_draft, part, nc,
        cta_part, plan.ctas_per_bb, plan.n_tiles, draft_bias, p_tok, lse, ref_max, ref_sum, flags,
        state);
  }
  return check_launch();
}

size_t dspark_verify_lmhead_workspace_size(int V, int r, int B, int K, int dm,
                                           int64_t n_target_rows) {
  (void)r;
  if (V <= 0 || B < 0 || K < 0 || dm <= 0 || n_target_rows < 0) return 0;
  return lm_ws(V, r, B, K, dm, n_target_rows).total;
}

dspark_status dspark_verify_lmhead(const void* hidden, const void* lm_head, int dm,
                                   int64_t n_target_rows, const int64_t* row_start,
                                   const int32_t* verify_len, const float* base_logits,
                                   const void* U, const void* W, dspark_dtype uw_dtype, int V,
                                   int r, int B, int K, const int32_t* prev_token,
                                   const float* inv_temp, const int32_t* tokens,
                                   const float* p_tok, const float* ref_max, const float* ref_sum,
                                   const float* draft_bias, const float* u_accept,
                                   const float* u_resample, int32_t* n_accepted,
                                   int32_t* out_tokens, int32_t* last_token, void* workspace,
                                   size_t ws_bytes, void* stream) {
  dspark_status st = check_shapes(V, r, B, K, uw_dtype);
  if (st != DSPARK_OK) return st;
  if (dm <= 0 || n_target_rows < 0) return DSPARK_ERR_INVALID_ARG;
  if (dm % 64 != 0 || dm > kLhMaxDm) return DSPARK_ERR_UNSUPPORTED;
  if (!workspace || !aligned(workspace, 256) ||
      ws_bytes < dspark_verify_lmhead_workspace_size(V, r, B, K, dm, n_target_rows))
    return DSPARK_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (B == 0) return clear_status(workspace, s);
  if (!hidden || !lm_head || n_target_rows <= 0 || !row_start || !verify_len || !base_logits ||
      !U || !W || !prev_token || !u_resample || !n_accepted || !out_tokens)
    return DSPARK_ERR_INVALID_ARG;
  if (K > 0 && (!tokens || !p_tok || !ref_max || !ref_sum || !u_accept))
    return DSPARK_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(lm_head, 16) || !aligned(base_logits, 16) ||
      !aligned(U, 16) || !aligned(W, 16) || (draft_bias && !aligned(draft_bias, 16)))
    return DSPARK_ERR_INVALID_ARG;
  if ((long long)B * (K + 1) > (1ll << 31) - 1 || n_target_rows > (1ll << 31) - 1)
    return DSPARK_ERR_UNSUPPORTED;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  if (uw_dtype == DSPARK_BF16)
    return verify_lmhead_impl<__nv_bfloat16>(hidden, lm_head, dm, n_target_rows, row_start,
                                             verify_len, base_logits, U, W, uw_dtype, V, r, B, K,
                                             prev_token, inv_temp, tokens, p_tok, ref_max, ref_sum,
                                             draft_bias, u_accept, u_resample, n_accepted,
                                             out_tokens, last_token, ws, s);
  return verify_lmhead_impl<float>(hidden, lm_head, dm, n_target_rows, row_start, verify_len,
                                   base_logits, U, W, uw_dtype, V, r, B, K, prev_token, inv_temp,
                                   tokens, p_tok, ref_max, ref_sum, draft_bias, u_accept,
                                   u_resample, n_accepted, out_tokens, last_token, ws, s);
}

dspark_status dspark_test_set_exchange_skew(int skew) {
  if (cudaDeviceSynchronize() != cudaSuccess) return DSPARK_ERR_CUDA;
  return cudaMemcpyToSymbol(g_test_exchange_skew, &skew, sizeof(int)) == cudaSuccess
             ? DSPARK_OK
             : DSPARK_ERR_CUDA;
}

dspark_status dspark_verify_noalloc_status(void* stream) {
  void* scratch = nullptr;
  const dspark_status st = noalloc_scratch(&scratch);
  if (st != DSPARK_OK) return st;
  return dspark_get_device_status(scratch, stream);
}

}  // extern "C"
