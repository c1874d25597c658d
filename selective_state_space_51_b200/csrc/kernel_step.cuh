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
// written once), as long as the per-channel arithmetic (convolution, softplus,
// two SiLUs, N exponentials) is not repeated by several threads: a thread
// owns a whole channel up to 16 states. The first thread of a channel writes
// the conv buffer and y after the readout is summed over the channel's
// threads by shuffles (N > 16 only).
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

// One thread per (b, e) channel and SPT consecutive states of it (QP threads
// per channel when N > SPT): the channel's scalars (conv, step size, gates)
// are computed once per thread, and its state group moves as SPT/4 16-byte
// accesses issued before any arithmetic. The grid's y index is the batch row,
// so no division is needed to find (b, e).
template <typename T, int SPT, int QP, bool VEC>
__device__ __forceinline__ void step_channel(const StepParams &p,
                                             const int64_t b) {
  const int64_t tx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int q = int(tx % QP);
  const int64_t e = tx / QP;
  const bool live = e < p.dim;
  const int64_t ch = b * p.dim + (live ? e : 0);
  const int N = p.dstate;
  const int n0 = SPT * q;
  const int K = p.conv_width;
  const T *Bm = static_cast<const T *>(p.B) + b * N;
  const T *Cm = static_cast<const T *>(p.C) + b * N;
  float *st = p.state + ch * N;

  // ---- the state group first
  float h[SPT];
  const bool vec = VEC && live && n0 + SPT <= N;
  if (vec) {
#pragma unroll
    for (int i = 0; i < SPT; i += 4) {
      const float4 v4 = *reinterpret_cast<const float4 *>(st + n0 + i);
      h[i] = v4.x; h[i + 1] = v4.y; h[i + 2] = v4.z; h[i + 3] = v4.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < SPT; ++i)
      h[i] = live && n0 + i < N ? st[n0 + i] : 0.0f;
  }

  // ---- the channel's input, through the causal convolution
  float xv = live ? Act<T>::load(static_cast<const T *>(p.x_new) + ch) : 0.0f;
  T *buf = nullptr;
  float acc = 0.0f;
  if (live && p.conv_state) {
    buf = static_cast<T *>(p.conv_state) + ch * K;
    acc = p.conv_bias ? p.conv_bias[e] : 0.0f;
#pragma unroll
    for (int j = 0; j < kMaxConvWidth; ++j)
      if (j < K)
        acc = fmaf(j + 1 < K ? Act<T>::load(buf + j + 1) : xv,
                   p.conv_weight[e * K + j], acc);
  }
  if (QP > 1) __syncwarp();  // the channel's threads have read the buffer
  if (buf) {
    if (q == 0) {
      // shift left by one sample and append; reads stay ahead of writes
#pragma unroll
      for (int j = 0; j < kMaxConvWidth; ++j)
        if (j < K)
          Act<T>::store(buf + j, j + 1 < K ? Act<T>::load(buf + j + 1) : xv);
    }
    xv = silu(acc);
  }

  float partial = 0.0f;
  if (live) {
    const float v = Act<T>::load(static_cast<const T *>(p.delta) + ch) +
                    (p.delta_bias ? p.delta_bias[e] : 0.0f);
    const float step = p.softplus ? softplus(v) : v;
    const float dx = step * xv;
    const float *al = p.A_log + e * N + n0;
#pragma unroll
    for (int i = 0; i < SPT; ++i) {
      if (n0 + i < N) {
        const float A = -expf(al[i]);
        const float zl = step * fmaxf(A * kLog2e, -FLT_MAX);
        const float a = ex2(zl);
        const float wf =
            p.write_zoh ? zoh_factor(step, zl, a, -expf(-al[i])) * xv : dx;
        h[i] = fmaf(a, h[i], wf * Act<T>::load(Bm + n0 + i));
        partial = fmaf(Act<T>::load(Cm + n0 + i), h[i], partial);
      }
    }
    if (vec) {
#pragma unroll
      for (int i = 0; i < SPT; i += 4)
        *reinterpret_cast<float4 *>(st + n0 + i) =
            make_float4(h[i], h[i + 1], h[i + 2], h[i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < SPT; ++i)
        if (n0 + i < N) st[n0 + i] = h[i];
    }
  }
  // sum the readout over the channel's QP threads
#pragma unroll
  for (int m = QP / 2; m > 0; m >>= 1)
    partial += __shfl_xor_sync(0xffffffffu, partial, m);
  if (live && q == 0) {
    float out = partial + (p.D ? p.D[e] * xv : 0.0f);
    if (p.z) out *= silu(Act<T>::load(static_cast<const T *>(p.z) + ch));
    Act<T>::store(static_cast<T *>(p.y) + ch, out);
  }
}

template <typename T, int SPT, int QP, bool VEC>
__global__ void __launch_bounds__(128) scan_step_kernel(const StepParams p) {
  for (int64_t b = blockIdx.y; b < p.batch; b += gridDim.y)
    step_channel<T, SPT, QP, VEC>(p, b);
}

}  // namespace ssm
