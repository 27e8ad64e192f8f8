// common.cuh -- device helpers shared by the DSpark kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include <mutex>

#include "../../include/dspark.h"

namespace dspark {

// ---------------------------------------------------------------------------
// host: per-device set-up
// ---------------------------------------------------------------------------

// Kernel attributes (the dynamic shared-memory limit) and device properties
// belong to one device: a process that drives several GPUs, or several host
// threads, must set them for every device it launches on, once.
constexpr int kMaxDevices = 64;
using DeviceOnce = std::once_flag[kMaxDevices];

inline int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) d = 0;
  return d;
}

// Runs f() once per device (the current one), thread-safe.
template <typename F>
inline void once_per_device(DeviceOnce& once, F&& f) {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) {
    f();
    return;
  }
  std::call_once(once[d], f);
}

// Maximum dynamic shared memory of a kernel, set once per device.
template <typename Kern>
inline void set_smem_once(DeviceOnce& once, Kern* kern, int bytes) {
  once_per_device(once, [&] {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
}

// Programmatic dependent launch.  grid_dep_wait blocks until the kernel
// before this one in the stream has completed and its writes are visible
// (it returns at once when this launch carries no programmatic dependency);
// grid_dep_launch lets a kernel launched behind this one with that
// dependency begin before this one ends.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launches kern<<<grid, block, smem, s>>>(args...) with programmatic stream
// serialisation: the kernel may start while the one before it in the stream
// runs (once every CTA of that one has called grid_dep_launch or exited),
// and orders itself behind it with grid_dep_wait.  Every kernel argument is
// passed explicitly (defaults do not apply through the pointer).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------------------
// sizes and workspace layout
// ---------------------------------------------------------------------------

// Rows of the vocabulary summarised by one softmax partial (one warp's rows).
constexpr int kChunk = 32;
// Elements of a target row reduced by one CTA in the target-statistics pass.
constexpr int kSeg = 8192;
// The workspace starts with a 2 KB header whose first word is the device
// status (DSPARK_FLAG_* bits); the persistent draft keeps its grid-barrier
// counters there.
constexpr size_t kHeaderBytes = 2048;
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline int n_chunks_of(int V) { return (V + kChunk - 1) / kChunk; }
__host__ __device__ inline int n_segs_of(int V) { return (V + kSeg - 1) / kSeg; }
__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Test hook of the timeout path (set by dspark_test_set_exchange_skew, 0
// in normal operation): when non-zero, the first record exchange of the
// persistent draft for one or two requests, and the partial-record exchange
// of the single-launch verify, wait for records that never arrive, so their
// bounded waits run out.  Read once per CTA.
static __device__ int g_test_exchange_skew;

// ---------------------------------------------------------------------------
// status word
// ---------------------------------------------------------------------------

__device__ __forceinline__ void raise_flag(unsigned* flags, unsigned f) { atomicOr(flags, f); }

// A token id read from memory, clamped into [0, V) (or -1 for "none" when
// allowed); an id outside the range raises DSPARK_FLAG_BAD_TOKEN.
__device__ __forceinline__ int checked_token(int x, int V, bool allow_none, unsigned* flags) {
  if (x < 0) {
    if (allow_none) return -1;
    raise_flag(flags, DSPARK_FLAG_BAD_TOKEN);
    return 0;
  }
  if (x >= V) {
    raise_flag(flags, DSPARK_FLAG_BAD_TOKEN);
    return allow_none ? -1 : V - 1;
  }
  return x;
}

// 1/T for request b; a non-positive or non-finite value raises
// DSPARK_FLAG_BAD_TEMP and is replaced by 1.
__device__ __forceinline__ float checked_inv_temp(const float* inv_temp, int b, unsigned* flags) {
  if (inv_temp == nullptr) return 1.0f;
  float it = inv_temp[b];
  if (!(it > 0.0f) || !isfinite(it)) {
    raise_flag(flags, DSPARK_FLAG_BAD_TEMP);
    return 1.0f;
  }
  return it;
}

// ---------------------------------------------------------------------------
// arithmetic
// ---------------------------------------------------------------------------

// 2^x on the SFU (relative error of a couple of ulp; subnormal results
// flush to zero, far below anything a sampling decision can see).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// An empty asm that takes v as an input: v is computed here, in program
// order, so every shared-memory load it was computed from has returned.  A
// warp that releases a buffer for an async-proxy refill (TMA, bulk copy)
// passes what it computed from its loads through here first, then syncs
// and arrives.  An arrive issued while the warp's loads were still in
// flight let the refill overwrite rows before they were read (measured: the
// first rows of a 128-row stage, read by the warps of lane quarters 0-1).
__device__ __forceinline__ void consumed(float v) { asm volatile("" ::"f"(v) : "memory"); }

// Softmax partial of a 32-row chunk of one request: A = max_j (bv_j + d_j),
// s = sum_j 2^(((bv_j - A) + d_j) * it2) (0 when every row is -inf), in four
// interleaved chains (row j in chain j % 4), combined as (c0 + c1) + (c2 + c3).
// bv - A is exact for the rows that carry the mass (Sterbenz).
__device__ __forceinline__ float2 chunk_partial32(const float (&bv)[32], const float (&d)[32],
                                                  float it2) {
  float A4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
  for (int j = 0; j < 32; ++j) A4[j & 3] = fmaxf(A4[j & 3], bv[j] + d[j]);
  const float A = fmaxf(fmaxf(A4[0], A4[1]), fmaxf(A4[2], A4[3]));
  float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int j = 0; j < 32; ++j) s4[j & 3] += ex2(((bv[j] - A) + d[j]) * it2);
  const float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
  return make_float2(A, A == -CUDART_INF_F ? 0.0f : sum);
}

// Merge softmax partial (A, s) into (M, S) (both relative to their own max).
__device__ __forceinline__ void merge_partial(float& M, float& S, float A, float s, float it2) {
  if (A == -CUDART_INF_F) return;
  const float Mn = fmaxf(M, A);
  S = S * ex2((M - Mn) * it2) + s * ex2((A - Mn) * it2);
  M = Mn;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// Inclusive prefix sum over the lanes of a warp (lane order), in fp64.
__device__ __forceinline__ double warp_incl_scan_d(double v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    double n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// ---------------------------------------------------------------------------
// loads
// ---------------------------------------------------------------------------

// 8 consecutive elements of a W / U row as fp32.  Row starts are 16-byte
// aligned (r % 8 == 0, base pointer 16-byte aligned).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&o)[8]) {
  uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
  o[0] = __uint_as_float(q.x << 16); o[1] = __uint_as_float(q.x & 0xffff0000u);
  o[2] = __uint_as_float(q.y << 16); o[3] = __uint_as_float(q.y & 0xffff0000u);
  o[4] = __uint_as_float(q.z << 16); o[5] = __uint_as_float(q.z & 0xffff0000u);
  o[6] = __uint_as_float(q.w << 16); o[7] = __uint_as_float(q.w & 0xffff0000u);
}
__device__ __forceinline__ void load8(const float* p, float (&o)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }

// L2 policy for data read exactly once (logit streams): evict first, so
// that it does not displace data that is re-read (W, partials).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// 128-bit streaming load with an L2 cache policy, not allocated in L1.
__device__ __forceinline__ float4 ld_stream4(const float* p, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0,%1,%2,%3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

// The transition bias U[x] . W[v] for one vocabulary row, accumulated in
// fp32 in ascending index order (fmaf).  The projection kernels and the
// samplers call this same function, so a re-computed chunk reproduces the
// projection's bias bit for bit on the CUDA-core path.
template <typename TW>
__device__ __forceinline__ float dot_row(const TW* __restrict__ wrow, const float* __restrict__ u, int r) {
  if constexpr (sizeof(TW) == 2) {
    if (r == 256) {
      // the whole 512-byte row in one round of loads, then the same
      // ascending-index FMA chain as the general loop below
      uint4 q[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) q[i] = __ldg(reinterpret_cast<const uint4*>(wrow) + i);
      float acc = 0.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float4 ua = *reinterpret_cast<const float4*>(u + 8 * i);
        const float4 ub = *reinterpret_cast<const float4*>(u + 8 * i + 4);
        acc = fmaf(__uint_as_float(q[i].x << 16), ua.x, acc);
        acc = fmaf(__uint_as_float(q[i].x & 0xffff0000u), ua.y, acc);
        acc = fmaf(__uint_as_float(q[i].y << 16), ua.z, acc);
        acc = fmaf(__uint_as_float(q[i].y & 0xffff0000u), ua.w, acc);
        acc = fmaf(__uint_as_float(q[i].z << 16), ub.x, acc);
        acc = fmaf(__uint_as_float(q[i].z & 0xffff0000u), ub.y, acc);
        acc = fmaf(__uint_as_float(q[i].w << 16), ub.z, acc);
        acc = fmaf(__uint_as_float(q[i].w & 0xffff0000u), ub.w, acc);
      }
      return acc;
    }
  }
  float acc = 0.0f;
  for (int i0 = 0; i0 < r; i0 += 64) {
    // issue up to eight independent 16-byte loads before using any of them
    float w[8][8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (i0 + 8 * q < r) load8(wrow + i0 + 8 * q, w[q]);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (i0 + 8 * q >= r) break;
      const float4 ua = *reinterpret_cast<const float4*>(u + i0 + 8 * q);
      const float4 ub = *reinterpret_cast<const float4*>(u + i0 + 8 * q + 4);
      acc = fmaf(w[q][0], ua.x, acc); acc = fmaf(w[q][1], ua.y, acc);
      acc = fmaf(w[q][2], ua.z, acc); acc = fmaf(w[q][3], ua.w, acc);
      acc = fmaf(w[q][4], ub.x, acc); acc = fmaf(w[q][5], ub.y, acc);
      acc = fmaf(w[q][6], ub.z, acc); acc = fmaf(w[q][7], ub.w, acc);
    }
  }
  return acc;
}

// ---------------------------------------------------------------------------
// block-wide reductions / scans over 256 threads (8 warps)
// ---------------------------------------------------------------------------

template <int NT>
__device__ __forceinline__ float block_max(float v, float* sh) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  float r = (lane < NT / 32) ? sh[lane] : -CUDART_INF_F;
  return warp_max(r);
}

template <int NT>
__device__ __forceinline__ double block_sum_d(double v, double* sh) {
  v = warp_sum_d(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  double r = (lane < NT / 32) ? sh[lane] : 0.0;
  return warp_sum_d(r);
}

// Exclusive prefix sum over the threads of a block (thread order), fp64.
// The result is non-decreasing in thread order when every v >= 0 (each
// value is a rounded running sum, never "inclusive minus v").
// Returns the exclusive prefix; *total receives the block total.
template <int NT>
__device__ __forceinline__ double block_excl_scan_d(double v, double* sh, double* total) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double incl = warp_incl_scan_d(v);
  double ex = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) ex = 0.0;
  __syncthreads();
  if (lane == 31) sh[w] = incl;
  __syncthreads();
  double wpre = 0.0;
  for (int i = 0; i < w; ++i) wpre += sh[i];
  double tot = 0.0;
  for (int i = 0; i < NT / 32; ++i) tot += sh[i];
  *total = tot;
  return (lane == 0) ? wpre : wpre + ex;
}

}  // namespace dspark
