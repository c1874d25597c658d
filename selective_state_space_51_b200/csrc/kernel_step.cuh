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
// written once), as long as neither the per-channel arithmetic (convolution,
// softplus, two SiLUs) nor the per-channel constants are redone per state
// group or per batch row: a thread owns a whole channel up to 16 states and
// keeps its constants in registers across the batch rows it walks. The first
// thread of a channel writes the conv buffer and y after the readout is
// summed over the channel's threads by shuffles (N > 16 only).
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

// Four consecutive activations as floats (one 8- or 16-byte load).
template <typename T>
__device__ __forceinline__ void load4(const T *p, float *out);
template <>
__device__ __forceinline__ void load4<float>(const float *p, float *out) {
  const float4 v = *reinterpret_cast<const float4 *>(p);
  out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p,
                                                     float *out) {
  const uint2 v = *reinterpret_cast<const uint2 *>(p);
  out[0] = __uint_as_float(v.x << 16);
  out[1] = __uint_as_float(v.x & 0xffff0000u);
  out[2] = __uint_as_float(v.y << 16);
  out[3] = __uint_as_float(v.y & 0xffff0000u);
}

// One thread per channel e and SPT consecutive states of it (QP threads per
// channel when N > SPT). The channel's constants (A log2 e, filter taps,
// biases, D) are loaded once into registers, and the thread then walks the
// batch rows b = blockIdx.y, blockIdx.y + gridDim.y, ...: per row the state
// group moves as SPT/4 16-byte accesses issued before any arithmetic, and
// the channel's scalars (convolution, step size, gates) are computed once.
// VEC: N % 4 == 0 and the state, B and C allow 4-element vector accesses.
// Shared memory per 128-thread block: each thread's A log2(e) (SPT floats) and
// filter taps (kMaxConvWidth floats), in rows padded by 4 words so that the
// 16-byte reads of 8 consecutive threads fall in distinct banks. Each thread
// reads back only its own rows, so no barrier is needed.
template <int SPT>
struct StepSmem {
  static constexpr int A_ROW = SPT + 4, W_ROW = kMaxConvWidth + 4;
  static constexpr int BYTES = 128 * (A_ROW + W_ROW) * 4;
};

// The vectorised kernels are held to 64 registers (8 blocks per SM): the step
// is latency-bound, and the extra resident warps keep more loads in flight.
template <typename T, int SPT, int QP, bool VEC>
__global__ void __launch_bounds__(128, VEC ? 8 : 1)
    scan_step_kernel(const StepParams p) {
  extern __shared__ __align__(16) float step_smem[];
  const int64_t tx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int q = int(tx % QP);
  const int64_t e = tx / QP;
  const bool live = e < p.dim;
  const int64_t es = live ? e : 0;
  const int N = p.dstate;
  const int n0 = SPT * q;
  const int K = p.conv_width;
  const bool vec = VEC && n0 + SPT <= N;

  // ---- the channel's constants, once, into this thread's shared rows
  float *const A2 = step_smem + threadIdx.x * StepSmem<SPT>::A_ROW;
  float *const cw = step_smem + 128 * StepSmem<SPT>::A_ROW +
                    threadIdx.x * StepSmem<SPT>::W_ROW;
#pragma unroll
  for (int i = 0; i < SPT; ++i)
    A2[i] = live && n0 + i < N
                ? fmaxf(-expf(p.A_log[es * N + n0 + i]) * kLog2e, -FLT_MAX)
                : 0.0f;
  float cbias = 0.0f;
#pragma unroll
  for (int j = 0; j < kMaxConvWidth; ++j)
    cw[j] = (p.conv_state && live && j < K) ? p.conv_weight[es * K + j] : 0.0f;
  if (p.conv_state && live) cbias = p.conv_bias ? p.conv_bias[es] : 0.0f;
  const float dbias = (live && p.delta_bias) ? p.delta_bias[es] : 0.0f;
  const float Dv = (live && p.D) ? p.D[es] : 0.0f;

  for (int64_t b = blockIdx.y; b < p.batch; b += gridDim.y) {
    const int64_t ch = b * p.dim + es;
    float *st = p.state + ch * N;

    // ---- the state group first
    float h[SPT];
    if (live && vec) {
#pragma unroll
      for (int i = 0; i < SPT; i += 4) {
        // the state is read once and written once per step: streaming
        // (evict-first) accesses
        const float4 v4 = __ldcs(reinterpret_cast<const float4 *>(st + n0 + i));
        h[i] = v4.x; h[i + 1] = v4.y; h[i + 2] = v4.z; h[i + 3] = v4.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < SPT; ++i)
        h[i] = live && n0 + i < N ? st[n0 + i] : 0.0f;
    }

    // ---- the channel's input, through the causal convolution
    float xv =
        live ? Act<T>::load(static_cast<const T *>(p.x_new) + ch) : 0.0f;
    T *buf = nullptr;
    float acc = cbias;
    if (live && p.conv_state) {
      buf = static_cast<T *>(p.conv_state) + ch * K;
      // the taps as two 16-byte reads of this thread's row
      const float4 w0 = *reinterpret_cast<const float4 *>(cw);
      const float4 w1 = *reinterpret_cast<const float4 *>(cw + 4);
      const float taps[kMaxConvWidth] = {w0.x, w0.y, w0.z, w0.w,
                                         w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int j = 0; j < kMaxConvWidth; ++j)
        if (j < K)
          acc = fmaf(j + 1 < K ? Act<T>::load(buf + j + 1) : xv, taps[j], acc);
    }
    if (QP > 1) __syncwarp();  // the channel's threads have read the buffer
    if (buf) {
      if (q == 0) {
        // shift left by one sample and append; reads stay ahead of writes
#pragma unroll
        for (int j = 0; j < kMaxConvWidth; ++j)
          if (j < K)
            Act<T>::store(buf + j,
                          j + 1 < K ? Act<T>::load(buf + j + 1) : xv);
      }
      xv = silu(acc);
    }

    float partial = 0.0f;
    if (live) {
      const float v =
          Act<T>::load(static_cast<const T *>(p.delta) + ch) + dbias;
      const float step = p.softplus ? softplus(v) : v;
      const float dx = step * xv;
      const T *Bm = static_cast<const T *>(p.B) + b * N + n0;
      const T *Cm = static_cast<const T *>(p.C) + b * N + n0;
#pragma unroll
      for (int i0 = 0; i0 < SPT; i0 += 4) {
        float Bv[4], Cv[4];
        if (vec) {
          load4<T>(Bm + i0, Bv);
          load4<T>(Cm + i0, Cv);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            Bv[i] = n0 + i0 + i < N ? Act<T>::load(Bm + i0 + i) : 0.0f;
            Cv[i] = n0 + i0 + i < N ? Act<T>::load(Cm + i0 + i) : 0.0f;
          }
        }
        const float4 a4 = *reinterpret_cast<const float4 *>(A2 + i0);
        const float Aq[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = i0 + i;
          if (n0 + k < N) {
            const float zl = step * Aq[i];
            const float a = sizeof(T) == 4 ? retention_f32(zl) : ex2(zl);
            const float wf =
                p.write_zoh
                    ? zoh_factor(step, zl, a,
                                 -expf(-p.A_log[es * N + n0 + k])) * xv
                    : dx;
            h[k] = fmaf(a, h[k], wf * Bv[i]);
            partial = fmaf(Cv[i], h[k], partial);
          }
        }
      }
      if (vec) {
#pragma unroll
        for (int i = 0; i < SPT; i += 4)
          __stcs(reinterpret_cast<float4 *>(st + n0 + i),
                 make_float4(h[i], h[i + 1], h[i + 2], h[i + 3]));
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
      float out = partial + Dv * xv;
      if (p.z) out *= silu(Act<T>::load(static_cast<const T *>(p.z) + ch));
      Act<T>::store(static_cast<T *>(p.y) + ch, out);
    }
  }
}

}  // namespace ssm
