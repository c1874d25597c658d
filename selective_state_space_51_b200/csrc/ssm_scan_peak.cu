// Measured rate of the SFU's exp2 (MUFU.EX2), the unit the scan's roofline
// divides by: a kernel whose threads do nothing but chains of ex2.approx.ftz.
#include <cuda_runtime.h>

#include "../../include/ssm_scan.h"
#include "device_math.cuh"

namespace {

constexpr int kChains = 8;    // independent chains per thread
constexpr int kUnroll = 4;    // chain steps per loop iteration

// x <- 2^(-x) keeps every value in (0.5, 1): one MUFU op per step, the
// negation folded into the instruction's operand.
__global__ void __launch_bounds__(256) ex2_rate_kernel(int iters,
                                                       float *sink) {
  float a[kChains];
#pragma unroll
  for (int j = 0; j < kChains; ++j)
    a[j] = 0.25f + 0.01f * float((threadIdx.x + j) & 15);
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
#pragma unroll
      for (int j = 0; j < kChains; ++j) a[j] = ssm::ex2(-a[j]);
  }
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < kChains; ++j) s += a[j];
  if (s == 1234.5f) sink[0] = s;  // keeps the chains live; never true
}

}  // namespace

extern "C" int ssm_measure_ex2_rate(int device, double *ex2_per_second) {
  if (!ex2_per_second) return SSM_ERR_INVALID;
  *ex2_per_second = 0.0;
  int count = 0, prev = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (device < 0 || device >= count) return SSM_ERR_INVALID;
  int sms = 0;
  if (cudaGetDevice(&prev) != cudaSuccess || cudaSetDevice(device) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) !=
          cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  int rc = SSM_OK;
  float *sink = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  const int threads = 256, blocks = sms * 8;  // 2048 threads per SM
  const int iters = 4096;
  if (cudaMalloc(&sink, sizeof(float)) != cudaSuccess ||
      cudaEventCreate(&e0) != cudaSuccess ||
      cudaEventCreate(&e1) != cudaSuccess) {
    cudaGetLastError();
    rc = SSM_ERR_CUDA;
  }
  if (rc == SSM_OK) {
    ex2_rate_kernel<<<blocks, threads>>>(iters / 8, sink);  // warm-up
    cudaEventRecord(e0);
    const int reps = 5;
    for (int r = 0; r < reps; ++r)
      ex2_rate_kernel<<<blocks, threads>>>(iters, sink);
    cudaEventRecord(e1);
    float ms = 0.0f;
    if (cudaEventSynchronize(e1) != cudaSuccess ||
        cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess || ms <= 0.0f) {
      cudaGetLastError();
      rc = SSM_ERR_CUDA;
    } else {
      const double ops = double(reps) * blocks * threads * double(iters) *
                         kUnroll * kChains;
      *ex2_per_second = ops / (double(ms) * 1e-3);
    }
  }
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (sink) cudaFree(sink);
  cudaSetDevice(prev);
  return rc;
}
