// ssm_scan_fwd_static_scratch: the forward pass for callers that cannot
// allocate device memory. It allocates nothing: the workspace that split
// sequences need lives in one fixed device array of this library, below.
//
// Some callers cannot call cudaMalloc. Examples are code that runs after a
// serving engine has handed all device memory to its own pool, or a plug-in
// whose host forbids allocation once its memory budget is fixed. cudaMalloc and
// cudaFree can also synchronize the whole device. The handle-based entry point
// may grow a workspace with cudaMallocAsync when it splits a sequence. This
// one uses the fixed array instead, and asks nothing of the allocator.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/ssm_scan.h"
#include "kernel_chunked.cuh"

namespace {

// Fixed scratch for split sequences: [0, 256) control words (status, launch
// ticket), then publication flags, then three float32 state arrays of
// batch x pieces x channels x states each. Every GPU that loads the library
// holds these bytes until the process exits.
constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
constexpr unsigned kSpinLimit = 1000u * 1000u;  // about one second of polls

struct DeviceScratch {
  unsigned char *ptr = nullptr;  // device address of g_scratch
  int sm_count = 0;
  unsigned epoch = 0;            // tag of the last call's publications
};
std::mutex g_lock;
DeviceScratch g_dev[kMaxDevices];

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

bool aligned(const void *p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// Same tile shapes as the handle-based entry point, one time block per
// channel.
using bf16 = __nv_bfloat16;
//                          T      NG TB  K  TW NW pad PB BFPB
using S16b = ssm::ChunkCfg<bf16,  4, 1, 4, 32, 4, 16, 0, 0>;
using S16f = ssm::ChunkCfg<float, 4, 1, 4, 16, 4, 16, 0, 0>;
using S8b = ssm::ChunkCfg<bf16,   2, 1, 2, 32, 4, 32, 0, 0>;
using S8f = ssm::ChunkCfg<float,  2, 1, 2, 16, 4, 32, 0, 0>;
using S4f = ssm::ChunkCfg<float,  1, 1, 1, 16, 4,  0, 0, 0>;

template <class Cfg, bool ZOH>
int run(DeviceScratch &d, ssm::ScanParams &p, int segments, int *status,
        cudaStream_t s) {
  const int64_t tiles = (p.dim + Cfg::G - 1) / Cfg::G;
  int64_t segs = segments;
  // Without a caller status word a given-up bounded wait could not be
  // reported, so such calls never split.
  if (!status) segs = 1;
  if (segs <= 0) {  // enough pieces to fill every resident block slot once
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, ssm::scan_chunked_kernel<Cfg, true, ZOH>, Cfg::THREADS,
            Cfg::SMEM_BYTES) != cudaSuccess) {
      cudaGetLastError();
      return SSM_ERR_CUDA;
    }
    const int64_t slots = int64_t(per_sm > 0 ? per_sm : 1) * d.sm_count;
    const int64_t base = p.batch * tiles;
    segs = base * 2 > slots ? 1 : slots / base;
    const int64_t max_segs = p.seqlen / (64 * Cfg::TW);
    if (segs > max_segs) segs = max_segs;
    if (segs < 1) segs = 1;
  }
  int64_t seg_len = p.seqlen;
  if (segs > 1) {
    const int64_t wins = (p.seqlen + Cfg::TW - 1) / Cfg::TW;
    seg_len = (wins + segs - 1) / segs * Cfg::TW;
    segs = (p.seqlen + seg_len - 1) / seg_len;
  }
  p.segments = int(segs);
  p.seg_len = seg_len;
  if (cudaFuncSetAttribute(ssm::scan_chunked_kernel<Cfg, true, ZOH>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Cfg::SMEM_BYTES) != cudaSuccess ||
      cudaFuncSetAttribute(ssm::scan_chunked_kernel<Cfg, false, ZOH>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Cfg::SMEM_BYTES) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (segs <= 1) {
    if (p.batch * tiles > 0x7fffffff) return SSM_ERR_UNSUPPORTED;
    ssm::scan_chunked_kernel<Cfg, false, ZOH>
        <<<unsigned(p.batch * tiles), Cfg::THREADS, Cfg::SMEM_BYTES, s>>>(p);
    return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
  }
  // carve the fixed array; reject problems it cannot hold
  const size_t nflags = size_t(p.batch) * segs * tiles;
  const size_t nstate = size_t(p.batch) * segs * p.dim * p.dstate;
  const size_t off_flags = 256;
  const size_t off_state = off_flags + round256(nflags * sizeof(unsigned));
  const size_t state_bytes = round256(nstate * sizeof(float));
  if (off_state + 3 * state_bytes > kScratchBytes) return SSM_ERR_UNSUPPORTED;
  if (segs * p.batch * tiles > 0x7fffffff) return SSM_ERR_UNSUPPORTED;
  unsigned char *base = d.ptr;
  p.flags = reinterpret_cast<unsigned *>(base + off_flags);
  p.agg_state = reinterpret_cast<float *>(base + off_state);
  p.agg_decay = reinterpret_cast<float *>(base + off_state + state_bytes);
  p.incl_state = reinterpret_cast<float *>(base + off_state + 2 * state_bytes);
  p.ticket = reinterpret_cast<unsigned *>(base + 4);
  p.status = status;
  p.spin_limit = kSpinLimit;
  p.debug = 0;
  // The array keeps the previous call's contents: the ticket restarts at
  // zero and this call's publication flags are cleared on the stream before
  // the launch (memsets, not allocations), so no flag of an earlier call can
  // be taken for this one's. The per-call tag is a second guard.
  if (++d.epoch >= (1u << 30)) d.epoch = 1;
  p.epoch = d.epoch;
  if (cudaMemsetAsync(p.ticket, 0, sizeof(unsigned), s) != cudaSuccess ||
      cudaMemsetAsync(p.flags, 0, nflags * sizeof(unsigned), s) !=
          cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  ssm::scan_chunked_kernel<Cfg, true, ZOH>
      <<<unsigned(segs * p.batch * tiles), Cfg::THREADS, Cfg::SMEM_BYTES, s>>>(
          p);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

template <bool ZOH>
int dispatch(DeviceScratch &d, ssm::ScanParams &p, int dtype, int segments,
             int *status, cudaStream_t s) {
  if (dtype == SSM_BF16) {
    if (p.dstate == 16) return run<S16b, ZOH>(d, p, segments, status, s);
    return run<S8b, ZOH>(d, p, segments, status, s);
  }
  if (p.dstate == 16) return run<S16f, ZOH>(d, p, segments, status, s);
  if (p.dstate == 8) return run<S8f, ZOH>(d, p, segments, status, s);
  return run<S4f, ZOH>(d, p, segments, status, s);
}

}  // namespace

extern "C" {

int ssm_scan_fwd_static_scratch(int device, const void *x, const void *delta,
                                const float *A_log, const void *B,
                                const void *C, const float *D, const void *z,
                                const float *delta_bias, uint32_t flags,
                                const float *h0, void *y, float *h_last,
                                ssm_scan_dims dims, int dtype, int segments,
                                int *status, struct CUstream_st *stream) {
  // ---- host-side checks, before anything reaches the GPU
  if (!x || !delta || !A_log || !B || !C || !y) return SSM_ERR_INVALID;
  if (dims.batch <= 0 || dims.seqlen <= 0 || dims.dim <= 0 || dims.dstate <= 0)
    return SSM_ERR_INVALID;
  if (flags & ~uint32_t(SSM_DELTA_SOFTPLUS | SSM_WRITE_ZOH))
    return SSM_ERR_INVALID;
  if (segments < 0) return SSM_ERR_INVALID;
  // a split call reports a given-up wait through the caller's status word
  if (segments > 1 && !status) return SSM_ERR_INVALID;
  if (device < 0 || device >= kMaxDevices) return SSM_ERR_INVALID;
  if (dtype != SSM_F32 && dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  const int esz = dtype == SSM_F32 ? 4 : 2;
  if (dims.dstate != 4 && dims.dstate != 8 && dims.dstate != 16)
    return SSM_ERR_UNSUPPORTED;
  if (dims.dstate * esz < 16 || (dims.dim * esz) % 16 != 0)
    return SSM_ERR_UNSUPPORTED;
  int64_t rows = 0, acts = 0;
  if (__builtin_mul_overflow(dims.batch, dims.seqlen, &rows) ||
      __builtin_mul_overflow(rows, dims.dim, &acts) ||
      acts > (int64_t(1) << 56))
    return SSM_ERR_INVALID;
  const void *tiles[] = {x, delta, z, B, C};
  for (const void *t : tiles)
    if (t && !aligned(t, 16)) return SSM_ERR_ALIGN;
  if (!aligned(y, esz)) return SSM_ERR_ALIGN;
  const float *params[] = {A_log, D, delta_bias, h0, h_last};
  for (const float *q : params)
    if (q && !aligned(q, 4)) return SSM_ERR_ALIGN;
  if (status && !aligned(status, 4)) return SSM_ERR_ALIGN;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (cur != device) return SSM_ERR_INVALID;

  // ---- once per device, with it current: the array's device address
  DeviceScratch *d = &g_dev[device];
  {
    std::lock_guard<std::mutex> guard(g_lock);
    if (!d->ptr) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor,
                                 device) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor,
                                 device) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount,
                                 device) != cudaSuccess) {
        cudaGetLastError();
        return SSM_ERR_CUDA;
      }
      if (major != 10 || minor != 0) return SSM_ERR_ARCH;
      void *ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || !ptr) {
        cudaGetLastError();
        return SSM_ERR_CUDA;
      }
      if (cudaMemset(ptr, 0, kScratchBytes) != cudaSuccess ||
          cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return SSM_ERR_CUDA;
      }
      d->ptr = static_cast<unsigned char *>(ptr);
      d->sm_count = sms;
    }
  }

  ssm::ScanParams p{};
  p.x = x; p.delta = delta; p.A_log = A_log; p.B = B; p.C = C;
  p.D = D; p.z = z; p.delta_bias = delta_bias; p.h0 = h0;
  p.y = y; p.h_last = h_last;
  p.batch = dims.batch; p.seqlen = dims.seqlen; p.dim = dims.dim;
  p.dstate = int(dims.dstate);
  p.softplus = (flags & SSM_DELTA_SOFTPLUS) ? 1 : 0;
  p.write_zoh = (flags & SSM_WRITE_ZOH) ? 1 : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  std::lock_guard<std::mutex> guard(g_lock);  // the epoch and the array
  return p.write_zoh ? dispatch<true>(*d, p, dtype, segments, status, s)
                     : dispatch<false>(*d, p, dtype, segments, status, s);
}

}  // extern "C"
