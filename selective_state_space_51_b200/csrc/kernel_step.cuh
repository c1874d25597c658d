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
  // bulk-copy variant only: device status word (kStepTimeout on a wait that
  // gave up) and the polls a wait makes before giving up
  int *status;
  unsigned spin_limit;
  // bulk-copy variant: per 128-channel column, a counter of the batch rows
  // handed out so far (zero before the launch); blocks of a column take rows
  // from it as they go, so the ones that run faster take more rows. nullptr:
  // block y takes rows y, y + gridDim.y, ...
  unsigned *row_counter;
};

// Device status written by the bulk-copy decode step (same word as the
// scan's status; 1 = a bounded wait gave up).
constexpr int kStepTimeout = 1;
// Polls of the final wait for copies still in flight after a wait gave up
// (independent of the caller's limit, which may be tiny in tests).
constexpr unsigned kStepDrainPolls = 1u << 22;

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


// ---------------------------------------------------------------------------
// Decode step with every per-row input and output moved by bulk copies.
// A block owns 128 consecutive channels and walks batch rows b = blockIdx.y,
// blockIdx.y + gridDim.y, ... For one row, everything the block reads is a
// handful of contiguous runs: its channels' [128 x N] float32 state, their
// x, raw step and z values, their [128 x K] conv buffers, and the row's B and
// C. Each run arrives in shared memory as one bulk copy (cp.async.bulk from
// this GPU's own memory; completion counted on an mbarrier), and the updated
// state, conv buffers and y leave the same way. Three buffers rotate over the
// rows, so the copies of the next two rows are in flight while one row is
// updated, and the state moves as whole cache lines.
// A thread owns one channel (N = 4, 8 or 16 states, N/4 16-byte chunks of
// its shared row). Its chunks are visited in an order rotated by its place in
// the quarter warp, so the 16-byte shared accesses of 8 consecutive threads
// fall in distinct banks. Every wait on an mbarrier is bounded; a wait that
// gives up sets the status word, and the block stops after draining its
// copies.
constexpr int kStepBulkBufs = 3;

template <typename T, int N>
struct StepBulkLayout {
  static constexpr int ESZ = sizeof(T);
  static constexpr int STATE = 0;
  static constexpr int X = 128 * N * 4;
  static constexpr int DL = X + 128 * ESZ;
  static constexpr int Z = DL + 128 * ESZ;
  static constexpr int Y = Z + 128 * ESZ;
  static constexpr int CONV = Y + 128 * ESZ;
  static constexpr int BM = CONV + 128 * kMaxConvWidth * ESZ;
  static constexpr int CM = BM + (N * ESZ + 15) / 16 * 16;
  static constexpr int BUF = CM + (N * ESZ + 15) / 16 * 16;  // one buffer
  static constexpr int BAR = kStepBulkBufs * BUF;            // mbarriers
  static constexpr int BYTES = BAR + 8 * kStepBulkBufs;
  static_assert(BUF % 16 == 0 && X % 16 == 0 && CONV % 16 == 0,
                "bulk copy destinations are 16-byte aligned");
};

__device__ __forceinline__ unsigned smem_addr(const void *p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

// Bounded wait for phase `parity` of an mbarrier; false if it gave up.
__device__ __forceinline__ bool mbar_wait(unsigned bar, unsigned parity,
                                          unsigned limit) {
  for (unsigned i = 0; i < limit; ++i) {
    unsigned done;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void bulk_load(unsigned dst, const void *src,
                                          unsigned bytes, unsigned bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_store(void *dst, unsigned src,
                                           unsigned bytes) {
  asm volatile(
      "cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
      "r"(src), "r"(bytes)
      : "memory");
}

template <typename T, int N>
__global__ void __launch_bounds__(128)
    scan_step_bulk_kernel(const StepParams p) {
  static_assert(N == 4 || N == 8 || N == 16, "whole 16-byte chunks");
  using Lay = StepBulkLayout<T, N>;
  constexpr int R = N / 4;  // 16-byte chunks per channel
  constexpr int NB = kStepBulkBufs;
  extern __shared__ __align__(128) unsigned char bulk_smem[];
  const unsigned sbase = smem_addr(bulk_smem);
  const unsigned bar0 = sbase + Lay::BAR;
  const int tid = threadIdx.x;
  const int64_t E = p.dim;
  const int64_t e0 = (int64_t)blockIdx.x * 128;
  const int nch = int(E - e0 < 128 ? E - e0 : 128);
  const bool live = tid < nch;
  const int64_t es = live ? e0 + tid : e0;
  const int K = p.conv_state ? p.conv_width : 0;
  constexpr int ESZ = Lay::ESZ;
  // run sizes of one row (all multiples of 16 bytes: checked on the host)
  const unsigned st_bytes = unsigned(nch) * N * 4;
  const unsigned act_bytes = unsigned(nch) * ESZ;
  const unsigned conv_bytes = unsigned(nch) * K * ESZ;
  constexpr unsigned bc_bytes = N * ESZ;
  const unsigned row_bytes = st_bytes + (p.z ? 3 : 2) * act_bytes +
                             conv_bytes + 2 * bc_bytes;
  // chunk k of this thread's row is visited at position (k - rot) mod R
  const int rot = ((tid & 7) * R / 8) % R;

  // ---- the channel's constants, in registers
  float A2[N];
#pragma unroll
  for (int i = 0; i < N; ++i)
    A2[i] = live ? fmaxf(-expf(p.A_log[es * N + i]) * kLog2e, -FLT_MAX) : 0.0f;
  float cw[kMaxConvWidth];
#pragma unroll
  for (int j = 0; j < kMaxConvWidth; ++j)
    cw[j] = (live && j < K) ? p.conv_weight[es * K + j] : 0.0f;
  const float cbias = (live && K && p.conv_bias) ? p.conv_bias[es] : 0.0f;
  const float dbias = (live && p.delta_bias) ? p.delta_bias[es] : 0.0f;
  const float Dv = (live && p.D) ? p.D[es] : 0.0f;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < NB; ++i)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8 * i)
                   : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const T *gx = static_cast<const T *>(p.x_new);
  const T *gdl = static_cast<const T *>(p.delta);
  const T *gz = static_cast<const T *>(p.z);
  const T *gB = static_cast<const T *>(p.B);
  const T *gC = static_cast<const T *>(p.C);
  T *gy = static_cast<T *>(p.y);
  T *gconv = static_cast<T *>(p.conv_state);

  // issue the copies of batch row b into buffer `buf` (thread 0)
  auto load_row = [&](int64_t b, int buf) {
    const unsigned d = sbase + buf * Lay::BUF;
    const unsigned bar = bar0 + 8 * buf;
    const int64_t ch = b * E + e0;
    asm volatile(
        "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
        "r"(row_bytes)
        : "memory");
    bulk_load(d + Lay::STATE, p.state + ch * N, st_bytes, bar);
    bulk_load(d + Lay::X, gx + ch, act_bytes, bar);
    bulk_load(d + Lay::DL, gdl + ch, act_bytes, bar);
    if (gz) bulk_load(d + Lay::Z, gz + ch, act_bytes, bar);
    if (K) bulk_load(d + Lay::CONV, gconv + ch * K, conv_bytes, bar);
    bulk_load(d + Lay::BM, gB + b * N, bc_bytes, bar);
    bulk_load(d + Lay::CM, gC + b * N, bc_bytes, bar);
  };

  // The batch row of each of this block's rows in flight, by buffer: taken
  // from the column's counter (or the fixed stride) when its copies are
  // issued; a row past the batch means there are no more.
  __shared__ long long s_row[NB];
  const int64_t first = blockIdx.y, stride = gridDim.y;
  unsigned *const counter =
      p.row_counter ? p.row_counter + blockIdx.x : nullptr;
  int64_t next_static = first;
  auto take_row = [&]() -> int64_t {
    if (counter) return int64_t(atomicAdd(counter, 1u));
    const int64_t r = next_static;
    next_static += stride;
    return r;
  };
  if (tid == 0)
    for (int i = 0; i < NB - 1; ++i) {
      const int64_t r = take_row();
      s_row[i] = r;
      if (r < p.batch) load_row(r, i);
    }
  __syncthreads();
  int64_t k = 0;
  bool failed = false;
  for (;; ++k) {
    const int buf = int(k % NB);
    const int64_t b = s_row[buf];
    if (b >= p.batch) break;  // the same value for every thread
    unsigned char *const B0 = bulk_smem + buf * Lay::BUF;
    // the copies of the row after next go into the buffer the previous row
    // used, once the stores that read it have finished reading
    if (tid == 0) {
      const int nb = int((k + NB - 1) % NB);
      const int64_t r = take_row();
      s_row[nb] = r;
      if (r < p.batch) {
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        load_row(r, nb);
      }
    }
    const bool ok =
        mbar_wait(bar0 + 8 * buf, unsigned(k / NB) & 1u, p.spin_limit);
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }

    if (live) {
      // ---- the channel's input, through the causal convolution
      float xv = Act<T>::load(reinterpret_cast<const T *>(B0 + Lay::X) + tid);
      if (K) {
        T *cb = reinterpret_cast<T *>(B0 + Lay::CONV) + tid * K;
        float hist[kMaxConvWidth];
#pragma unroll
        for (int j = 0; j < kMaxConvWidth; ++j)
          hist[j] = j + 1 < K ? Act<T>::load(cb + j + 1) : xv;
        float acc = cbias;
#pragma unroll
        for (int j = 0; j < kMaxConvWidth; ++j)
          if (j < K) acc = fmaf(hist[j], cw[j], acc);
        // shift left by one sample and append
#pragma unroll
        for (int j = 0; j < kMaxConvWidth; ++j)
          if (j < K) Act<T>::store(cb + j, hist[j]);
        xv = silu(acc);
      }
      const float v =
          Act<T>::load(reinterpret_cast<const T *>(B0 + Lay::DL) + tid) +
          dbias;
      const float step = p.softplus ? softplus(v) : v;
      const float dx = step * xv;
      const T *Bm = reinterpret_cast<const T *>(B0 + Lay::BM);
      const T *Cm = reinterpret_cast<const T *>(B0 + Lay::CM);
      float *const row = reinterpret_cast<float *>(B0 + Lay::STATE) + tid * N;
      float partial = 0.0f;
#pragma unroll
      for (int c = 0; c < R; ++c) {
        const int j = R == 1 ? 0 : (c + rot) % R;  // this visit's chunk
        const int i0 = 4 * j;
        float Bv[4], Cv[4];
        load4<T>(Bm + i0, Bv);
        load4<T>(Cm + i0, Cv);
        const float4 h4 = *reinterpret_cast<const float4 *>(row + i0);
        float hq[4] = {h4.x, h4.y, h4.z, h4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          // A2[i0 + i] with i0 a runtime chunk: select from the registers
          float Ai = A2[i];
#pragma unroll
          for (int jj = 1; jj < R; ++jj)
            if (j == jj) Ai = A2[4 * jj + i];
          const float zl = step * Ai;
          const float a = sizeof(T) == 4 ? retention_f32(zl) : ex2(zl);
          const float wf =
              p.write_zoh
                  ? zoh_factor(step, zl, a, -expf(-p.A_log[es * N + i0 + i])) *
                        xv
                  : dx;
          hq[i] = fmaf(a, hq[i], wf * Bv[i]);
          partial = fmaf(Cv[i], hq[i], partial);
        }
        *reinterpret_cast<float4 *>(row + i0) =
            make_float4(hq[0], hq[1], hq[2], hq[3]);
      }
      float out = partial + Dv * xv;
      if (gz)
        out *= silu(Act<T>::load(reinterpret_cast<const T *>(B0 + Lay::Z) +
                                 tid));
      Act<T>::store(reinterpret_cast<T *>(B0 + Lay::Y) + tid, out);
    }
    // this thread's shared writes become visible to the copy engine, then
    // one thread stores the updated runs
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      const unsigned d = sbase + buf * Lay::BUF;
      const int64_t ch = b * E + e0;
      bulk_store(p.state + ch * N, d + Lay::STATE, st_bytes);
      bulk_store(gy + ch, d + Lay::Y, act_bytes);
      if (K) bulk_store(gconv + ch * K, d + Lay::CONV, conv_bytes);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
  }
  if (tid == 0) {
    if (failed) {
      atomicExch(p.status, kStepTimeout);
      // copies still in flight (rows k .. k + NB - 1 may have been issued)
      // land before the block's memory is released; these waits are
      // bounded too
      for (int64_t r = k; r < k + NB; ++r)
        if (s_row[r % NB] < p.batch)
          mbar_wait(bar0 + 8 * int(r % NB), unsigned(r / NB) & 1u,
                    kStepDrainPolls);
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
}

}  // namespace ssm
