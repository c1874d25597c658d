// Batched decode step: one new token for each of `batch` sequences, updating
// the conv buffer and the state in place.
//
// Page "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
// (www.abhik.ai/papers/mamba), section "Original paper, equations and
// runnable CPU code", row "6. Carry both buffers to the next token": shift
// the K-sample conv buffer and append the new input; x = SiLU(sum_k buf[k]
// w[k] + bias) (row "4. Add causal local context before selecting
// coefficients"); delta = softplus(raw + bias); state = exp(delta A) state +
// delta B x; y = sum_n C state + D x; y *= SiLU(z).
//
// The step is bound by memory traffic on the [b, E, N] float32 state (read and
// written once). A thread owns (b, e, one group of up to 4 states): its state
// group is one 16-byte access, and consecutive threads touch consecutive
// groups, so a warp moves whole contiguous rows. The threads of a channel
// (QP of them, a power of two) recompute the channel's scalars (conv, step,
// gate) from cached loads; the first one writes the conv buffer and y after
// the readout is summed over the group by shuffles.
#pragma once

#include <float.h>

#include "device_math.cuh"

namespace ssm {

struct StepParams {
  const void *x_new;       // [b, E]
  void *conv_state;        // [b, E, K] or nullptr
  const float *conv_weight;  // [E, K]
  const float *conv_bias;  // [E] or nullptr
  int conv_width;          // K
  const void *delta;       // [b, E]
  const float *delta_bias;  // [E] or nullptr
  const float *A_log;      // [E, N]
  const void *B;           // [b, N]
  const void *C;           // [b, N]
  const float *D;          // [E] or nullptr
  const void *z;           // [b, E] or nullptr
  float *state;            // [b, E, N]
  void *y;                 // [b, E]
  int64_t batch, dim;
  int dstate;
  int softplus, write_zoh;
};

constexpr int kMaxConvWidth = 8;

template <typename T, int QP, bool VEC>
__global__ void __launch_bounds__(256) scan_step_kernel(const StepParams p) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int q = int(gid % QP);                 // state group of this thread
  const int64_t ch = gid / QP;                 // (b, e)
  const bool live = ch < p.batch * p.dim;
  const int64_t b = live ? ch / p.dim : 0;
  const int64_t e = live ? ch - b * p.dim : 0;
  const int N = p.dstate;
  const int n0 = 4 * q;
  const T *xn = static_cast<const T *>(p.x_new);
  const T *dl = static_cast<const T *>(p.delta);
  const T *zz = static_cast<const T *>(p.z);
  const T *Bm = static_cast<const T *>(p.B);
  const T *Cm = static_cast<const T *>(p.C);

  // the channel's input: the new sample, through the causal convolution
  float xv = live ? Act<T>::load(xn + ch) : 0.0f;
  float win[kMaxConvWidth];
  const int K = p.conv_width;
  T *buf = nullptr;
  if (live && p.conv_state) {
    buf = static_cast<T *>(p.conv_state) + ch * K;
#pragma unroll
    for (int k = 0; k < kMaxConvWidth; ++k)
      if (k < K) win[k] = (k + 1 < K) ? Act<T>::load(buf + k + 1) : xv;
  }
  // every thread of a channel has read the old buffer before its first
  // thread overwrites it (all lanes reach this barrier)
  __syncwarp();
  if (buf) {
    float acc = p.conv_bias ? p.conv_bias[e] : 0.0f;
#pragma unroll
    for (int k = 0; k < kMaxConvWidth; ++k)
      if (k < K) acc = fmaf(win[k], p.conv_weight[e * K + k], acc);
    if (q == 0) {
#pragma unroll
      for (int k = 0; k < kMaxConvWidth; ++k)
        if (k < K) Act<T>::store(buf + k, win[k]);
    }
    xv = silu(acc);
  }
  float partial = 0.0f;
  if (live) {
    const float v = Act<T>::load(dl + ch) + (p.delta_bias ? p.delta_bias[e] : 0.0f);
    const float step = p.softplus ? softplus(v) : v;
    const float dx = step * xv;
    float *st = p.state + ch * N;
    // a whole group of 4 states moves as one 16-byte access when it can
    const bool vec = VEC && n0 + 4 <= N;
    float h4[4];
    if (vec) {
      const float4 v4 = *reinterpret_cast<const float4 *>(st + n0);
      h4[0] = v4.x; h4[1] = v4.y; h4[2] = v4.z; h4[3] = v4.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) h4[i] = n0 + i < N ? st[n0 + i] : 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int n = n0 + i;
      if (n < N) {
        const float al = p.A_log[e * N + n];
        const float zl = step * fmaxf(-expf(al) * kLog2e, -FLT_MAX);
        const float a = ex2(zl);
        const float wf = p.write_zoh ? zoh_factor(step, zl, a, -expf(-al)) * xv : dx;
        h4[i] = fmaf(a, h4[i], wf * Act<T>::load(Bm + b * N + n));
        partial = fmaf(Act<T>::load(Cm + b * N + n), h4[i], partial);
      }
    }
    if (vec) {
      *reinterpret_cast<float4 *>(st + n0) = make_float4(h4[0], h4[1], h4[2], h4[3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (n0 + i < N) st[n0 + i] = h4[i];
    }
  }
  // sum the readout over the channel's QP threads
#pragma unroll
  for (int m = QP / 2; m > 0; m >>= 1)
    partial += __shfl_xor_sync(0xffffffffu, partial, m);
  if (live && q == 0) {
    float out = partial + (p.D ? p.D[e] * xv : 0.0f);
    if (zz) out *= silu(Act<T>::load(zz + ch));
    Act<T>::store(static_cast<T *>(p.y) + ch, out);
  }
}

}  // namespace ssm
