// Sequential variant: one thread per (batch, channel) walks the whole
// sequence, keeping that channel's N states in float32 registers. It runs any
// shape (any E, any L, N up to 64) and serves as the general path for shapes
// the chunked variant does not tile.
//
// Recurrence (page "Mamba: Linear-Time Sequence Modeling with Selective State
// Spaces", www.abhik.ai/papers/mamba, section "Original paper, equations and
// runnable CPU code", rows 1, 2 and 5): delta = softplus(raw + bias);
// a = exp(delta * A) with A = -exp(A_log); h = a * h + delta * B * x;
// y = sum_n C * h + D * x, read after the update; y *= SiLU(z). With the
// exact zero-order-hold flag the write is expm1(delta A) / A * B * x. With a
// convolution (row "4. Add causal local context before selecting
// coefficients") x is SiLU of the causal depthwise convolution of the input,
// zeros before the first step.
#pragma once

#include <float.h>

#include "device_math.cuh"
#include "scan_params.cuh"

namespace ssm {

template <typename T, int NMAX>
__global__ void __launch_bounds__(128)
scan_sequential_kernel(const ScanParams p) {
  const int64_t pair = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (pair >= p.batch * p.dim) return;
  const int64_t b = pair / p.dim;
  const int64_t e = pair - b * p.dim;
  const int N = p.dstate;
  const int64_t L = p.seqlen, E = p.dim;

  float A2[NMAX];  // A * log2(e), so that a = 2^(delta * A2)
  float iA[NMAX];  // 1 / A (exact zero-order-hold write only)
  float h[NMAX];
#pragma unroll
  for (int n = 0; n < NMAX; ++n) {
    A2[n] = 0.0f;
    iA[n] = 0.0f;
    h[n] = 0.0f;
    if (n < N) {
      // clamp so that a zero step never meets -inf (0 * -inf = NaN)
      A2[n] = fmaxf(-expf(p.A_log[e * N + n]) * kLog2e, -FLT_MAX);
      iA[n] = -expf(-p.A_log[e * N + n]);
      if (p.h0) h[n] = p.h0[(b * E + e) * N + n];
    }
  }
  // convolution taps right-aligned to the newest input; win holds the
  // previous kScanConvMaxWidth - 1 inputs, oldest first
  const bool conv = p.conv_weight != nullptr;
  float cw[kScanConvMaxWidth] = {};
  float win[kScanConvMaxWidth - 1] = {};
  float cbias = 0.0f;
  if (conv) {
#pragma unroll
    for (int k = 0; k < kScanConvMaxWidth; ++k) {
      const int kk = k - (kScanConvMaxWidth - p.conv_width);
      cw[k] = kk >= 0 ? p.conv_weight[e * p.conv_width + kk] : 0.0f;
    }
    cbias = p.conv_bias ? p.conv_bias[e] : 0.0f;
  }
  const float bias = p.delta_bias ? p.delta_bias[e] : 0.0f;
  const float Dv = p.D ? p.D[e] : 0.0f;
  const T *x = static_cast<const T *>(p.x);
  const T *dl = static_cast<const T *>(p.delta);
  const T *z = static_cast<const T *>(p.z);
  const T *Bm = static_cast<const T *>(p.B);
  const T *Cm = static_cast<const T *>(p.C);
  T *y = static_cast<T *>(p.y);

  for (int64_t t = 0; t < L; ++t) {
    const int64_t i = (b * L + t) * E + e;
    const int64_t r = (b * L + t) * N;
    const float v = Act<T>::load(dl + i) + bias;
    const float step = p.softplus ? softplus(v) : v;
    float xv = Act<T>::load(x + i);
    if (conv) {
      float acc = cbias;
#pragma unroll
      for (int k = 0; k < kScanConvMaxWidth - 1; ++k)
        acc = fmaf(cw[k], win[k], acc);
      acc = fmaf(cw[kScanConvMaxWidth - 1], xv, acc);
#pragma unroll
      for (int k = 0; k + 1 < kScanConvMaxWidth - 1; ++k) win[k] = win[k + 1];
      win[kScanConvMaxWidth - 2] = xv;
      xv = silu(acc);
    }
    const float dx = step * xv;
    float acc = 0.0f;
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
      if (n < N) {
        const float zl = step * A2[n];
        const float a = sizeof(T) == 4 ? retention_f32(zl) : ex2(zl);
        const float wf = p.write_zoh ? zoh_factor(step, zl, a, iA[n]) * xv : dx;
        h[n] = fmaf(a, h[n], wf * Act<T>::load(Bm + r + n));
        acc = fmaf(Act<T>::load(Cm + r + n), h[n], acc);
      }
    }
    acc = fmaf(Dv, xv, acc);
    if (z) acc *= silu(Act<T>::load(z + i));
    Act<T>::store(y + i, acc);
  }
  if (p.h_last) {
#pragma unroll
    for (int n = 0; n < NMAX; ++n)
      if (n < N) p.h_last[(b * E + e) * N + n] = h[n];
  }
}

}  // namespace ssm
