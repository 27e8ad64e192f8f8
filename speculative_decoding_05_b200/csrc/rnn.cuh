// rnn.cuh -- the RNN sequential head's state update.
//
// freeaitool.com, "DeepSeek DSpark complete guide", 3.1: besides the Markov
// head the sequential head can be an RNN head that keeps a recurrent state
// and so captures longer dependencies (the page gives no formula).  Reading
// taken: an Elman recurrence in the rank-r space of the Markov head's
// lookup, whose input is that lookup:
//     s_{-1} = h0[b] (zeros without h0),  x_{-1} = prev_token[b]
//     s_k    = tanh(R s_{k-1} + U[x_{k-1}])
//     bias_k = s_k . W^T      (then the Markov head's softmax and sampling)
// p_d(x_k | x_<k) stays a single softmax, exact, as the verify needs.
//
// Per position the draft runs rnn_state_kernel (this file), the tensor-core
// projection with the state as operand A, and the two-level sampler.  The
// state is kept in fp32; operand A holds it as two bf16 rows, high part
// h = bf16(s) and low part l = bf16(s - h), both multiplied by the same W
// block, so the projection sees s to about 2^-17 relative.
#pragma once

#include "common.cuh"

namespace dspark {

constexpr int kRnnThreads = 256;

// One CTA per request: s_k from s_{k-1} (state, or h0 at k = 0) and the
// previous token; writes the state in place (fp32), its split rows
// [B, 2r] bf16 (operand A of the projection) and, if asked, states[b, k, :].
template <typename TW>
__global__ void __launch_bounds__(kRnnThreads)
rnn_state_kernel(const TW* __restrict__ U, const TW* __restrict__ R, int V, int r, int K, int k,
                 const int32_t* __restrict__ prev_token, const int32_t* __restrict__ tokens,
                 const float* __restrict__ h0, float* __restrict__ state,
                 __nv_bfloat16* __restrict__ a_rows, float* __restrict__ states_out,
                 unsigned* flags) {
  // the projection of this position may begin launching (its producers
  // read only W and the base logits; the rest of it waits for this kernel)
  grid_dep_launch();
  extern __shared__ float s_prev[];  // [r]
  const int b = blockIdx.x;
  int x = (k == 0) ? prev_token[b] : tokens[(size_t)b * K + (k - 1)];
  x = checked_token(x, V, k == 0, flags);
  for (int i = threadIdx.x; i < r; i += blockDim.x)
    s_prev[i] = (k == 0) ? (h0 != nullptr ? h0[(size_t)b * r + i] : 0.0f) : state[(size_t)b * r + i];
  __syncthreads();
  for (int i = threadIdx.x; i < r; i += blockDim.x) {
    const TW* rrow = R + (size_t)i * r;
    float acc = 0.0f;
    for (int j = 0; j < r; ++j) acc = fmaf(to_f32(rrow[j]), s_prev[j], acc);
    if (x >= 0) acc += to_f32(U[(size_t)x * r + i]);
    const float sv = tanhf(acc);
    state[(size_t)b * r + i] = sv;
    const __nv_bfloat16 hi = __float2bfloat16_rn(sv);
    const __nv_bfloat16 lo = __float2bfloat16_rn(sv - __bfloat162float(hi));
    a_rows[(size_t)b * 2 * r + i] = hi;
    a_rows[(size_t)b * 2 * r + r + i] = lo;
    if (states_out != nullptr) states_out[((size_t)b * K + k) * r + i] = sv;
  }
}

}  // namespace dspark
