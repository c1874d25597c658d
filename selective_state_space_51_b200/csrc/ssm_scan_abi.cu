// C ABI of libssmscan.so: handle management, host-side validation, variant
// choice and launches. Declarations and the contract live in
// include/ssm_scan.h.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <new>

#include "../../include/ssm_scan.h"
#include "kernel_bwd.cuh"
#include "kernel_chunked.cuh"
#include "kernel_sequential.cuh"
#include "kernel_step.cuh"

constexpr unsigned kDefaultSpinLimit = 1000u * 1000u;  // ~1 s of polls

struct ssm_scan_s {
  int device = 0;
  int sm_count = 0;
  int variant = SSM_VARIANT_AUTO;
  int segments = 0;
  int time_blocks = 0;
  int last_variant = 0;
  int last_segments = 0;
  unsigned epoch = 0;
  unsigned debug = 0;
  unsigned spin_limit = kDefaultSpinLimit;
  // control block (device, kCtlBytes): [0] status word, [1] launch ticket,
  // from [kCtlRowCounters] the decode step's per-column row counters
  int *ctl = nullptr;
  // split-sequence workspace: flags, then three state arrays
  void *ws = nullptr;
  size_t ws_bytes = 0;
  // backward: the forward's state checkpoints
  float *ckpt = nullptr;
  size_t ckpt_bytes = 0;
  // what ckpt holds, when ckpt_saved: the checkpoints of the last forward
  // with SSM_SAVE_CHECKPOINTS, for this shape, dtype and flags
  bool ckpt_saved = false;
  // deterministic backward: the per-block partial sums
  float *det = nullptr;
  size_t det_bytes = 0;
  // persistent-block backward: hand-over flags and carried sums
  void *bdyn = nullptr;
  size_t bdyn_bytes = 0;
  ssm_scan_dims ckpt_dims{};
  int ckpt_dtype = 0;
  uint32_t ckpt_flags = 0;
};

namespace {

bool aligned(const void *p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

bool mul_ok(int64_t a, int64_t b, int64_t *out) {
  return !__builtin_mul_overflow(a, b, out);
}

template <typename T, int NMAX>
int launch_sequential(const ssm::ScanParams &p, cudaStream_t s) {
  const int64_t pairs = p.batch * p.dim;
  const int threads = 128;
  const int64_t blocks = (pairs + threads - 1) / threads;
  if (blocks > 0x7fffffff) return SSM_ERR_UNSUPPORTED;
  ssm::scan_sequential_kernel<T, NMAX><<<(unsigned)blocks, threads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

template <typename T>
int dispatch_sequential(const ssm::ScanParams &p, cudaStream_t s) {
  if (p.dstate <= 4) return launch_sequential<T, 4>(p, s);
  if (p.dstate <= 8) return launch_sequential<T, 8>(p, s);
  if (p.dstate <= 16) return launch_sequential<T, 16>(p, s);
  if (p.dstate <= 32) return launch_sequential<T, 32>(p, s);
  return launch_sequential<T, 64>(p, s);
}

// Chunked-variant shapes. Paddings (bytes: per tile row, per block of rows,
// per block of float B/C rows) make each lane access pattern bank-conflict
// free for that lane layout.
using bf16 = __nv_bfloat16;
//                          T      NG TB  K  TW NW pad  PB  BFPB
using C16b1 = ssm::ChunkCfg<bf16,  4, 1, 4, 32, 4, 16,  0,  0>;
using C16f1 = ssm::ChunkCfg<float, 4, 1, 4, 16, 4, 16,  0,  0>;
using C16b2 = ssm::ChunkCfg<bf16,  4, 2, 8, 32, 4,  0, 16, 64>;
using C16f2 = ssm::ChunkCfg<float, 4, 2, 8, 16, 4, 32, 16, 64>;
using C8b1 = ssm::ChunkCfg<bf16,   2, 1, 2, 32, 4, 32,  0,  0>;
using C8f1 = ssm::ChunkCfg<float,  2, 1, 2, 16, 4, 32,  0,  0>;
using C8b2 = ssm::ChunkCfg<bf16,   2, 2, 8, 32, 4,  0, 16, 32>;
using C8f2 = ssm::ChunkCfg<float,  2, 2, 8, 16, 4, 32, 64, 32>;
using C4f1 = ssm::ChunkCfg<float,  1, 1, 1, 16, 4,  0,  0,  0>;
using C4f2 = ssm::ChunkCfg<float,  1, 2, 8, 16, 4,  0, 64, 16>;
// 16-channel tiles for the specialised bfloat16 path: twice the blocks, so
// the last wave's imbalance over the SMs is about half as large
using C16b1h = ssm::ChunkCfg<bf16, 4, 1, 4, 32, 2, 16,  0,  0>;

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Size of the handle's control block, and the word where the decode step's
// row counters (one per 128-channel column) start.
constexpr int kCtlBytes = 4096;
constexpr int kCtlRowCounters = 4;
constexpr int kMaxRowCounters = kCtlBytes / 4 - kCtlRowCounters;

// The checkpoint workspace, grown on `s` to at least `need` bytes.
int ensure_ckpt(ssm_scan_s *h, size_t need, cudaStream_t s) {
  if (need <= h->ckpt_bytes) return SSM_OK;
  if (h->ckpt) cudaFreeAsync(h->ckpt, s);
  h->ckpt = nullptr;
  h->ckpt_bytes = 0;
  h->ckpt_saved = false;
  if (cudaMallocAsync(reinterpret_cast<void **>(&h->ckpt), need, s) !=
      cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_NOMEM;
  }
  h->ckpt_bytes = need;
  return SSM_OK;
}

// Checkpoint floats of a (batch, seqlen, dim, dstate) scan: one state every
// kCkptSteps steps; false on overflow.
bool ckpt_floats(const ssm_scan_dims &d, int64_t *out) {
  int64_t bd = 0, st = 0;
  const int64_t nck = (d.seqlen + ssm::kCkptSteps - 1) / ssm::kCkptSteps;
  return mul_ok(d.batch, d.dim, &bd) && mul_ok(bd, d.dstate, &st) &&
         mul_ok(st, nck, out) && *out <= (int64_t(1) << 56);
}

// The handle's control block ([0] status word, [1] launch ticket, then the
// decode step's row counters), made on first use on `s`.
int ensure_ctl(ssm_scan_s *h, cudaStream_t s) {
  if (h->ctl) return SSM_OK;
  if (cudaMallocAsync(reinterpret_cast<void **>(&h->ctl), kCtlBytes, s) !=
      cudaSuccess) {
    cudaGetLastError();
    h->ctl = nullptr;
    return SSM_ERR_NOMEM;
  }
  return cudaMemsetAsync(h->ctl, 0, kCtlBytes, s) == cudaSuccess
             ? SSM_OK
             : SSM_ERR_CUDA;
}

// Grow the split workspace for `segs` pieces; fills the ScanParams pointers.
int ensure_workspace(ssm_scan_s *h, ssm::ScanParams &p, int64_t tiles,
                     int64_t segs, cudaStream_t s) {
  const size_t nflags = size_t(p.batch) * segs * tiles;
  const size_t nstate = size_t(p.batch) * segs * p.dim * p.dstate;
  const size_t off_state = align256(nflags * sizeof(unsigned));
  const size_t bytes = off_state + 3 * align256(nstate * sizeof(float));
  {
    const int rc = ensure_ctl(h, s);
    if (rc != SSM_OK) return rc;
  }
  if (bytes > h->ws_bytes) {
    if (h->ws) cudaFreeAsync(h->ws, s);
    h->ws = nullptr;
    h->ws_bytes = 0;
    if (cudaMallocAsync(&h->ws, bytes, s) != cudaSuccess) {
      cudaGetLastError();
      return SSM_ERR_NOMEM;
    }
    if (cudaMemsetAsync(h->ws, 0, bytes, s) != cudaSuccess) return SSM_ERR_CUDA;
    h->ws_bytes = bytes;
    h->epoch = 0;
  }
  if (++h->epoch >= (1u << 30)) h->epoch = 1;
  unsigned char *base = static_cast<unsigned char *>(h->ws);
  const size_t sz = align256(nstate * sizeof(float));
  p.flags = reinterpret_cast<unsigned *>(base);
  p.agg_state = reinterpret_cast<float *>(base + off_state);
  p.agg_decay = reinterpret_cast<float *>(base + off_state + sz);
  p.incl_state = reinterpret_cast<float *>(base + off_state + 2 * sz);
  p.status = h->ctl;
  p.ticket = reinterpret_cast<unsigned *>(h->ctl + 1);
  p.epoch = h->epoch;
  p.spin_limit = h->spin_limit;
  p.debug = h->debug;
  // The launch ticket restarts at zero and this call's publication flags are
  // cleared on the stream before the launch, so a flag left by an earlier
  // call (or an earlier replay of a captured graph) is never taken for one of
  // this call's; the per-call tag is a second guard for eager calls.
  if (cudaMemsetAsync(p.ticket, 0, sizeof(unsigned), s) != cudaSuccess ||
      cudaMemsetAsync(p.flags, 0, nflags * sizeof(unsigned), s) !=
          cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  return SSM_OK;
}

// Pieces per sequence: enough that the blocks fill every resident slot once,
// each piece at least 64 windows long (so the start-up replay after the
// look-back stays a small fraction), and 1 when channels alone fill the GPU.
template <class Cfg, bool ZOH, bool CONV>
int64_t auto_segments(const ssm::ScanParams &p, int sm_count) {
  static int per_sm = 0;  // resident blocks per SM for this shape
  if (!per_sm) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, ssm::scan_chunked_kernel<Cfg, true, ZOH, CONV>, Cfg::THREADS,
            Cfg::SMEM_BYTES) != cudaSuccess) {
      cudaGetLastError();
      n = 1;
    }
    per_sm = n > 0 ? n : 1;
  }
  const int64_t tiles = (p.dim + Cfg::G - 1) / Cfg::G;
  const int64_t base = p.batch * tiles;
  const int64_t slots = int64_t(per_sm) * sm_count;
  if (base * 2 > slots) return 1;
  const int64_t max_segs = p.seqlen / (64 * Cfg::TW);
  int64_t segs = slots / base;
  if (segs > max_segs) segs = max_segs;
  return segs < 2 ? 1 : segs;
}

template <class Cfg, bool SPLIT, bool ZOH, bool CONV, bool FAST = false,
          bool CKPT = false, bool SAVE = false, bool DYN = false>
int launch_kernel(const ssm::ScanParams &p, int64_t blocks, cudaStream_t s) {
  if (blocks > 0x7fffffff) return SSM_ERR_UNSUPPORTED;
  auto kern =
      ssm::scan_chunked_kernel<Cfg, SPLIT, ZOH, CONV, FAST, CKPT, SAVE, DYN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Cfg::SMEM_BYTES) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  kern<<<(unsigned)blocks, Cfg::THREADS, Cfg::SMEM_BYTES, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// Whether the specialised scan of these arguments runs on persistent blocks:
// when its tiles do not divide evenly over the schedulers (16 warps per SM),
// blocks take chunks of them in ticket order, so that every scheduler
// carries the same work, where one block per tile would leave some of them
// a fifth warp to the end. On yes, sets the chunking in p, grows and clears
// the hand-over workspace and returns the worker count in *workers (else 0).
template <class Cfg>
int plan_dyn(ssm_scan_s *h, ssm::ScanParams &p, int64_t tiles,
             cudaStream_t s, int64_t *workers) {
  *workers = 0;
  const int64_t w = int64_t(h->sm_count) * (16 / Cfg::NW);
  const int64_t units = p.batch * tiles;
  const bool force = (h->debug & ssm::kDebugForceDyn) != 0;
  const int64_t chunk = force ? ssm::kDynTestChunk : ssm::kDynChunk;
  if (h->segments > 0 || (h->debug & ssm::kDebugNoDyn) ||
      chunk % Cfg::TW != 0 || p.seqlen <= chunk ||
      !(force || (units > w && units % w != 0)))
    return SSM_OK;
  const int64_t C = (p.seqlen + chunk - 1) / chunk;
  p.segments = int(C);
  p.seg_len = chunk;
  const int rc = ensure_workspace(h, p, tiles, C, s);
  if (rc != SSM_OK) return rc;
  *workers = std::min(w, units * C);
  return SSM_OK;
}

template <class Cfg, bool ZOH = false, bool CONV = false>
int launch_chunked(ssm_scan_s *h, ssm::ScanParams &p, int64_t segs_req,
                   cudaStream_t s) {
  const int64_t tiles = (p.dim + Cfg::G - 1) / Cfg::G;
  int64_t segs = segs_req > 0 ? segs_req
                              : auto_segments<Cfg, ZOH, CONV>(p, h->sm_count);
  int64_t seg_len = p.seqlen;
  if (segs > 1) {
    const int64_t wins = (p.seqlen + Cfg::TW - 1) / Cfg::TW;
    const int64_t per = (wins + segs - 1) / segs;
    seg_len = per * Cfg::TW;
    segs = (p.seqlen + seg_len - 1) / seg_len;
  }
  p.segments = int(segs);
  p.seg_len = seg_len;
  h->last_segments = int(segs);
  if constexpr (!ZOH && Cfg::TB == 1) {
    // whole tiles and windows, gated, softplus, no checkpoints: the
    // specialised kernel tests none of these at run time
    if (segs <= 1 && p.z && p.softplus && !p.ckpt && p.y &&
        p.dim % Cfg::G == 0 && p.seqlen % Cfg::TW == 0) {
      int64_t workers = 0;
      const int rc = plan_dyn<Cfg>(h, p, tiles, s, &workers);
      if (rc != SSM_OK) return rc;
      if (workers > 0)
        return launch_kernel<Cfg, false, false, CONV, true, false, false,
                             true>(p, workers, s);
      return launch_kernel<Cfg, false, false, CONV, true>(
          p, p.batch * tiles, s);
    }
  }
  if (segs <= 1)
    return launch_kernel<Cfg, false, ZOH, CONV>(p, p.batch * tiles, s);
  const int rc = ensure_workspace(h, p, tiles, segs, s);
  if (rc != SSM_OK) return rc;
  return launch_kernel<Cfg, true, ZOH, CONV>(p, segs * p.batch * tiles, s);
}

// Whether the chunked variant can run these arguments: N of 4, 8 or 16, whole
// 16-byte chunks per channel tile row and per B/C row, 16-byte aligned tiles.
bool chunked_supported(const ssm::ScanParams &p, int dtype) {
  const int esz = dtype == SSM_F32 ? 4 : 2;
  if (p.dstate != 4 && p.dstate != 8 && p.dstate != 16) return false;
  if (p.dstate * esz < 16) return false;
  if ((p.dim * esz) % 16 != 0) return false;
  const void *tiles[] = {p.x, p.delta, p.z, p.B, p.C};
  for (const void *t : tiles)
    if (t && !aligned(t, 16)) return false;
  return true;
}

// Time blocks per channel: 1. Where channels are few, sequences are split
// into pieces instead (see auto_segments), which keeps the cheaper
// one-lane-per-step arithmetic; 2 is available on request.
int auto_time_blocks(const ssm::ScanParams &, int) { return 1; }

template <class Cf1, class Cf2>
int pick(ssm_scan_s *h, ssm::ScanParams &p, int tb, int64_t segs,
         cudaStream_t s) {
  // the zero-order-hold write and the fused convolution run with one time
  // block
  if (p.conv_weight) {
    if (tb != 1) return SSM_ERR_UNSUPPORTED;
    return p.write_zoh ? launch_chunked<Cf1, true, true>(h, p, segs, s)
                       : launch_chunked<Cf1, false, true>(h, p, segs, s);
  }
  if (p.write_zoh)
    return tb == 1 ? launch_chunked<Cf1, true>(h, p, segs, s)
                   : SSM_ERR_UNSUPPORTED;
  if (tb == 1) return launch_chunked<Cf1>(h, p, segs, s);
  if (tb == 2) return launch_chunked<Cf2>(h, p, segs, s);
  return SSM_ERR_UNSUPPORTED;
}

int dispatch_chunked(ssm_scan_s *h, ssm::ScanParams &p, int dtype, int tb,
                     int64_t segs, cudaStream_t s) {
  if (dtype == SSM_BF16) {
    if (p.dstate == 16 && tb == 1 && segs <= 1 && !p.write_zoh && p.z &&
        p.softplus && !p.ckpt && p.dim % C16b1h::G == 0 &&
        p.seqlen % C16b1h::TW == 0 &&
        p.batch * (p.dim / C16b1h::G) >= 2 * int64_t(h->sm_count) * 4)
      return p.conv_weight ? launch_chunked<C16b1h, false, true>(h, p, 1, s)
                           : launch_chunked<C16b1h>(h, p, 1, s);
    if (p.dstate == 16) return pick<C16b1, C16b2>(h, p, tb, segs, s);
    if (p.dstate == 8) return pick<C8b1, C8b2>(h, p, tb, segs, s);
    return SSM_ERR_UNSUPPORTED;
  }
  if (p.dstate == 16) return pick<C16f1, C16f2>(h, p, tb, segs, s);
  if (p.dstate == 8) return pick<C8f1, C8f2>(h, p, tb, segs, s);
  if (p.dstate == 4) return pick<C4f1, C4f2>(h, p, tb, segs, s);
  return SSM_ERR_UNSUPPORTED;
}

// The forward with SSM_SAVE_CHECKPOINTS: unsplit, one time block, the
// checkpoints written into p.ckpt; the specialised instantiation where the
// scan path would take it.
template <class Cfg>
int launch_save(ssm_scan_s *h, ssm::ScanParams &p, cudaStream_t s) {
  const int64_t blocks = p.batch * ((p.dim + Cfg::G - 1) / Cfg::G);
  p.segments = 1;
  p.seg_len = p.seqlen;
  h->last_segments = 1;
  if (p.write_zoh) return launch_kernel<Cfg, false, true, false>(p, blocks, s);
  if (p.z && p.softplus && p.y && p.dim % Cfg::G == 0 &&
      p.seqlen % Cfg::TW == 0) {
    int64_t workers = 0;
    const int rc =
        plan_dyn<Cfg>(h, p, (p.dim + Cfg::G - 1) / Cfg::G, s, &workers);
    if (rc != SSM_OK) return rc;
    if (workers > 0)
      return launch_kernel<Cfg, false, false, false, true, false, true, true>(
          p, workers, s);
    return launch_kernel<Cfg, false, false, false, true, false, true>(
        p, blocks, s);
  }
  return launch_kernel<Cfg, false, false, false>(p, blocks, s);
}

int dispatch_save(ssm_scan_s *h, ssm::ScanParams &p, int dtype,
                  cudaStream_t s) {
  if (dtype == SSM_BF16) {
    if (p.dstate == 16) {
      if (p.dim % C16b1h::G == 0 && p.seqlen % C16b1h::TW == 0 &&
          p.batch * (p.dim / C16b1h::G) >= 2 * int64_t(h->sm_count) * 4)
        return launch_save<C16b1h>(h, p, s);
      return launch_save<C16b1>(h, p, s);
    }
    if (p.dstate == 8) return launch_save<C8b1>(h, p, s);
    return SSM_ERR_UNSUPPORTED;
  }
  if (p.dstate == 16) return launch_save<C16f1>(h, p, s);
  if (p.dstate == 8) return launch_save<C8f1>(h, p, s);
  if (p.dstate == 4) return launch_save<C4f1>(h, p, s);
  return SSM_ERR_UNSUPPORTED;
}

template <typename T, int SPT, int QP>
int launch_step_cfg(const ssm::StepParams &p, bool vec, int sm_count,
                    cudaStream_t s) {
  const int64_t threads = p.dim * QP;
  const int64_t bx = (threads + 127) / 128;
  if (bx > 0x7fffffff) return SSM_ERR_UNSUPPORTED;
  auto kern = vec ? ssm::scan_step_kernel<T, SPT, QP, true>
                  : ssm::scan_step_kernel<T, SPT, QP, false>;
  // one wave: as many batch-row strides as leave every block resident at
  // once (each thread walks batch / grid.y rows with its channel's
  // constants in registers), so no block starts late
  static int occupancy[2] = {0, 0};  // resident blocks per SM, per kernel
  int &per_sm = occupancy[vec ? 1 : 0];
  if (per_sm < 1) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, kern, 128, ssm::StepSmem<SPT>::BYTES) != cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = 1;
    }
    per_sm = n;
  }
  int64_t by = int64_t(sm_count) * per_sm / bx;
  if (by > p.batch) by = p.batch;
  if (by > 65535) by = 65535;
  if (by < 1) by = 1;
  const dim3 grid{static_cast<unsigned>(bx), static_cast<unsigned>(by), 1u};
  kern<<<grid, 128, ssm::StepSmem<SPT>::BYTES, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// The bulk-copy decode step (N = 4, 8 or 16): one 128-channel block per
// state run, grid.y batch-row strides sized so every block is resident.
template <typename T, int N>
int launch_step_bulk(const ssm::StepParams &p, int sm_count, cudaStream_t s) {
  const int64_t bx = (p.dim + 127) / 128;
  if (bx > 0x7fffffff) return SSM_ERR_UNSUPPORTED;
  auto kern = ssm::scan_step_bulk_kernel<T, N>;
  constexpr int smem = ssm::StepBulkLayout<T, N>::BYTES;
  static int per_sm = 0;  // resident blocks per SM
  if (per_sm < 1) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess) {
      cudaGetLastError();
      return SSM_ERR_CUDA;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, 128, smem) !=
            cudaSuccess ||
        n < 1) {
      cudaGetLastError();
      n = 1;
    }
    per_sm = n;
  }
  int64_t by = int64_t(sm_count) * per_sm / bx;
  if (by > p.batch) by = p.batch;
  if (by > 65535) by = 65535;
  if (by < 1) by = 1;
  // rows are handed out by the column's counter when there is one (cleared
  // here, on the launch's stream), else by a fixed stride
  if (p.row_counter &&
      cudaMemsetAsync(p.row_counter, 0, size_t(bx) * sizeof(unsigned), s) !=
          cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  const dim3 grid{static_cast<unsigned>(bx), static_cast<unsigned>(by), 1u};
  kern<<<grid, 128, smem, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// States per thread: the whole channel up to 16, else 16 per thread and 2 or
// 4 threads per channel.
template <typename T>
int launch_step(const ssm::StepParams &p, bool vec, int sms, cudaStream_t s) {
  if (p.dstate <= 4) return launch_step_cfg<T, 4, 1>(p, vec, sms, s);
  if (p.dstate <= 8) return launch_step_cfg<T, 8, 1>(p, vec, sms, s);
  if (p.dstate <= 16) return launch_step_cfg<T, 16, 1>(p, vec, sms, s);
  if (p.dstate <= 32) return launch_step_cfg<T, 16, 2>(p, vec, sms, s);
  return launch_step_cfg<T, 16, 4>(p, vec, sms, s);
}

// The forward scan behind both entry points; conv_weight == nullptr: x is
// the scan input as it is.
int scan_fwd(ssm_scan_s *h, const void *x, const float *conv_weight,
             const float *conv_bias, int conv_width, const void *delta,
             const float *A_log, const void *B, const void *C, const float *D,
             const void *z, const float *delta_bias, uint32_t flags,
             const float *h0, void *y, float *h_last, ssm_scan_dims dims,
             int dtype, cudaStream_t s) {
  // ---- host-side validation: nothing touches the GPU before it passes
  if (!h || !x || !delta || !A_log || !B || !C || !y) return SSM_ERR_INVALID;
  if (dims.batch <= 0 || dims.seqlen <= 0 || dims.dim <= 0 || dims.dstate <= 0)
    return SSM_ERR_INVALID;
  if (flags & ~uint32_t(SSM_DELTA_SOFTPLUS | SSM_WRITE_ZOH |
                        (conv_weight ? 0u : unsigned(SSM_SAVE_CHECKPOINTS))))
    return SSM_ERR_INVALID;
  if (conv_weight &&
      (conv_width < 1 || conv_width > ssm::kScanConvMaxWidth))
    return SSM_ERR_INVALID;
  if (dtype != SSM_F32 && dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if (dims.dstate > 64) return SSM_ERR_UNSUPPORTED;
  int64_t rows = 0, acts = 0, bc = 0, st = 0;
  if (!mul_ok(dims.batch, dims.seqlen, &rows) ||
      !mul_ok(rows, dims.dim, &acts) || !mul_ok(rows, dims.dstate, &bc) ||
      !mul_ok(dims.batch * dims.dim, dims.dstate, &st) ||
      acts > (int64_t(1) << 56))
    return SSM_ERR_INVALID;
  const size_t esz = dtype == SSM_F32 ? 4 : 2;
  const void *acts_in[] = {x, delta, B, C, z, y};
  for (const void *p : acts_in)
    if (p && !aligned(p, esz)) return SSM_ERR_ALIGN;
  const float *params[] = {A_log, D, delta_bias, h0, h_last, conv_weight,
                           conv_bias};
  for (const float *p : params)
    if (p && !aligned(p, 4)) return SSM_ERR_ALIGN;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (cur != h->device) return SSM_ERR_INVALID;

  ssm::ScanParams p{};
  p.x = x; p.delta = delta; p.A_log = A_log; p.B = B; p.C = C;
  p.D = D; p.z = z; p.delta_bias = delta_bias; p.h0 = h0;
  p.y = y; p.h_last = h_last;
  p.batch = dims.batch; p.seqlen = dims.seqlen; p.dim = dims.dim;
  p.dstate = (int)dims.dstate;
  p.softplus = (flags & SSM_DELTA_SOFTPLUS) ? 1 : 0;
  p.write_zoh = (flags & SSM_WRITE_ZOH) ? 1 : 0;
  p.conv_weight = conv_weight;
  p.conv_bias = conv_weight ? conv_bias : nullptr;
  p.conv_width = conv_weight ? conv_width : 0;
  p.segments = 1;

  const bool chunk_ok = chunked_supported(p, dtype);
  if (flags & SSM_SAVE_CHECKPOINTS) {
    // the training forward: unsplit chunked scan, checkpoints kept
    if (!chunk_ok || h->variant == SSM_VARIANT_SEQUENTIAL ||
        h->time_blocks > 1)
      return SSM_ERR_UNSUPPORTED;
    int64_t ck = 0;
    if (!ckpt_floats(dims, &ck)) return SSM_ERR_INVALID;
    int rc = ensure_ckpt(h, size_t(ck) * sizeof(float), s);
    if (rc != SSM_OK) return rc;
    h->ckpt_saved = false;
    p.ckpt = h->ckpt;
    rc = dispatch_save(h, p, dtype, s);
    if (rc != SSM_OK) return rc;
    h->ckpt_saved = true;
    h->ckpt_dims = dims;
    h->ckpt_dtype = dtype;
    h->ckpt_flags = flags & (SSM_DELTA_SOFTPLUS | SSM_WRITE_ZOH);
    h->last_variant = SSM_VARIANT_CHUNKED;
    return SSM_OK;
  }
  int variant = h->variant;
  if (variant == SSM_VARIANT_AUTO)
    variant = chunk_ok ? SSM_VARIANT_CHUNKED : SSM_VARIANT_SEQUENTIAL;
  int rc;
  if (variant == SSM_VARIANT_CHUNKED) {
    if (!chunk_ok) return SSM_ERR_UNSUPPORTED;
    const int tb = h->time_blocks ? h->time_blocks
                                  : auto_time_blocks(p, h->sm_count);
    rc = dispatch_chunked(h, p, dtype, tb, h->segments, s);
  } else if (dtype == SSM_F32) {
    rc = dispatch_sequential<float>(p, s);
  } else {
    rc = dispatch_sequential<__nv_bfloat16>(p, s);
  }
  if (rc == SSM_OK) {
    h->last_variant = variant;
    if (variant != SSM_VARIANT_CHUNKED) h->last_segments = 1;
  }
  return rc;
}

// ---- backward
// out = the fixed-order sum of `slices` arrays of n floats (n a multiple of
// 4), on `s`.
int sum_slices(const float *part, int64_t slices, int64_t n, float *out,
               cudaStream_t s) {
  const int64_t n4 = n / 4;
  const int64_t grid = std::min<int64_t>((n4 + 255) / 256, 4096);
  ssm::sum_slices_kernel<<<unsigned(grid < 1 ? 1 : grid), 256, 0, s>>>(
      part, slices, n, out);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// Two warps per block: the 2.8B layer shape's 1280 blocks then fill 148 SMs
// at 9 blocks each in one wave, with at most 9 blocks where 8.65 is the
// mean (4-warp blocks: 5 where the mean is 4.3).
constexpr int kBwdWarps = 2;

template <typename T, int NG, bool ZOH>
int launch_bwd(ssm_scan_s *h, ssm::BwdParams &p, cudaStream_t s) {
  using Cfg = ssm::BwdCfg<T, NG, kBwdWarps>;
  const int64_t tiles = (p.dim + Cfg::G - 1) / Cfg::G;
  const int64_t blocks = p.batch * tiles;
  if (blocks > 0x7fffffff) return SSM_ERR_UNSUPPORTED;
  // whole tiles and windows, gated, softplus: the specialised instantiation;
  // deterministic sums: per-block partials, then fixed-order reductions
  const bool fast = p.dim % Cfg::G == 0 && p.seqlen % Cfg::TW == 0 && p.z &&
                    p.softplus;
  const bool det = p.part_dB != nullptr;
  // persistent blocks where the tiles do not divide evenly over 16 warps per
  // SM (as in the forward): chunks of the sweep hand their state over
  int64_t grid = blocks;
  bool dyn = false;
  if (fast && !(h->debug & ssm::kDebugNoDyn)) {
    const bool force = (h->debug & ssm::kDebugForceDyn) != 0;
    const int64_t wc = (force ? ssm::kDynTestChunk : ssm::kDynChunk) / Cfg::TW;
    const int64_t nwin = p.seqlen / Cfg::TW;
    const int64_t workers = int64_t(h->sm_count) * (16 / kBwdWarps);
    if (wc > 0 && nwin > wc &&
        (force || (blocks > workers && blocks % workers != 0))) {
      const int64_t C = (nwin + wc - 1) / wc;
      const size_t nflags = size_t(p.batch) * C * tiles;
      const size_t off = align256(nflags * sizeof(unsigned));
      const size_t need =
          off + size_t(blocks) * Cfg::THREADS * 12 * sizeof(float);
      int rc = ensure_ctl(h, s);
      if (rc != SSM_OK) return rc;
      if (need > h->bdyn_bytes) {
        if (h->bdyn) cudaFreeAsync(h->bdyn, s);
        h->bdyn = nullptr;
        h->bdyn_bytes = 0;
        if (cudaMallocAsync(&h->bdyn, need, s) != cudaSuccess) {
          cudaGetLastError();
          return SSM_ERR_NOMEM;
        }
        h->bdyn_bytes = need;
      }
      unsigned char *base = static_cast<unsigned char *>(h->bdyn);
      p.dyn_flags = reinterpret_cast<unsigned *>(base);
      p.dyn_carry = reinterpret_cast<float *>(base + off);
      p.dyn_ticket = reinterpret_cast<unsigned *>(h->ctl + 1);
      p.dyn_chunks = int(C);
      p.dyn_chunk_windows = int(wc);
      p.status = h->ctl;
      p.spin_limit = h->spin_limit;
      p.debug = h->debug;
      // the ticket restarts and the hand-over flags are cleared on the
      // stream before every launch (graph replays included)
      if (cudaMemsetAsync(p.dyn_ticket, 0, sizeof(unsigned), s) !=
              cudaSuccess ||
          cudaMemsetAsync(p.dyn_flags, 0, nflags * sizeof(unsigned), s) !=
              cudaSuccess) {
        cudaGetLastError();
        return SSM_ERR_CUDA;
      }
      dyn = true;
      grid = std::min<int64_t>(workers, blocks * C);
    }
  }
  auto kern =
      dyn ? (det ? ssm::scan_bwd_kernel<T, NG, kBwdWarps, ZOH, true, true, true>
                 : ssm::scan_bwd_kernel<T, NG, kBwdWarps, ZOH, true, false,
                                        true>)
      : det
          ? (fast ? ssm::scan_bwd_kernel<T, NG, kBwdWarps, ZOH, true, true>
                  : ssm::scan_bwd_kernel<T, NG, kBwdWarps, ZOH, false, true>)
          : (fast ? ssm::scan_bwd_kernel<T, NG, kBwdWarps, ZOH, true, false>
                  : ssm::scan_bwd_kernel<T, NG, kBwdWarps, ZOH, false, false>);
  const int smem =
      Cfg::SMEM_BYTES + (det ? (kBwdWarps - 1) * ssm::kBwdRedBytes : 0);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  kern<<<unsigned(grid), Cfg::THREADS, smem, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return SSM_ERR_CUDA;
  if (!det) return SSM_OK;
  const int64_t bln = p.batch * p.seqlen * p.dstate;
  const int64_t en = p.dim * p.dstate;
  int rc = sum_slices(p.part_dB, tiles, bln, p.dB, s);
  if (rc == SSM_OK) rc = sum_slices(p.part_dC, tiles, bln, p.dC, s);
  if (rc == SSM_OK) rc = sum_slices(p.part_dA, p.batch, en, p.dA_log, s);
  if (rc == SSM_OK && p.dD)
    rc = sum_slices(p.part_dD, p.batch, p.dim, p.dD, s);
  if (rc == SSM_OK && p.ddelta_bias)
    rc = sum_slices(p.part_db, p.batch, p.dim, p.ddelta_bias, s);
  return rc;
}

// The training forward (checkpoints, no y) and the reverse sweep for one
// (forward config, activation type, states per lane); with `reuse`, the
// reverse sweep alone, from the checkpoints a SSM_SAVE_CHECKPOINTS forward
// left.
template <class Cf, typename T, int NG>
int run_bwd(ssm_scan_s *h, ssm::ScanParams &fp, ssm::BwdParams &bp,
            bool reuse, cudaStream_t s) {
  if (reuse)  // the training forward left the checkpoints
    return fp.write_zoh ? launch_bwd<T, NG, true>(h, bp, s)
                        : launch_bwd<T, NG, false>(h, bp, s);
  const int64_t tiles = (fp.dim + Cf::G - 1) / Cf::G;
  const int64_t blocks = fp.batch * tiles;
  // the checkpoint-only forward: no readout, C and z not read; with whole
  // tiles and windows and the softplus step, the specialised instantiation
  const bool fast = !fp.write_zoh && fp.softplus && fp.dim % Cf::G == 0 &&
                    fp.seqlen % Cf::TW == 0;
  int64_t workers = 0;
  int rc = SSM_OK;
  if (fast) rc = plan_dyn<Cf>(h, fp, tiles, s, &workers);
  if (rc != SSM_OK) return rc;
  rc = fp.write_zoh
           ? launch_kernel<Cf, false, true, false, false, true>(fp, blocks, s)
       : workers > 0
           ? launch_kernel<Cf, false, false, false, true, true, false, true>(
                 fp, workers, s)
       : fast
           ? launch_kernel<Cf, false, false, false, true, true>(fp, blocks, s)
           : launch_kernel<Cf, false, false, false, false, true>(fp, blocks,
                                                                s);
  if (rc != SSM_OK) return rc;
  return fp.write_zoh ? launch_bwd<T, NG, true>(h, bp, s)
                      : launch_bwd<T, NG, false>(h, bp, s);
}

}  // namespace

extern "C" {

int ssm_scan_step(ssm_scan_t h, const void *x_new, void *conv_state,
                  const float *conv_weight, const float *conv_bias,
                  int conv_width, const void *delta, const float *delta_bias,
                  const float *A_log, const void *B, const void *C,
                  const float *D, const void *z, uint32_t flags, float *state,
                  void *y, ssm_scan_dims dims, int dtype,
                  struct CUstream_st *stream) {
  if (!h || !x_new || !delta || !A_log || !B || !C || !state || !y)
    return SSM_ERR_INVALID;
  if (dims.batch <= 0 || dims.dim <= 0 || dims.dstate <= 0 || dims.seqlen != 1)
    return SSM_ERR_INVALID;
  if (flags & ~uint32_t(SSM_DELTA_SOFTPLUS | SSM_WRITE_ZOH))
    return SSM_ERR_INVALID;
  if (conv_state && (!conv_weight || conv_width < 1 ||
                     conv_width > ssm::kMaxConvWidth))
    return SSM_ERR_INVALID;
  if (dtype != SSM_F32 && dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if (dims.dstate > 64) return SSM_ERR_UNSUPPORTED;
  int64_t chans = 0, st = 0;
  if (!mul_ok(dims.batch, dims.dim, &chans) ||
      !mul_ok(chans, dims.dstate, &st) || st > (int64_t(1) << 56))
    return SSM_ERR_INVALID;
  const size_t esz = dtype == SSM_F32 ? 4 : 2;
  const void *acts[] = {x_new, conv_state, delta, B, C, z, y};
  for (const void *q : acts)
    if (q && !aligned(q, esz)) return SSM_ERR_ALIGN;
  const float *params[] = {conv_weight, conv_bias, delta_bias, A_log, D,
                           state};
  for (const float *q : params)
    if (q && !aligned(q, 4)) return SSM_ERR_ALIGN;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (cur != h->device) return SSM_ERR_INVALID;

  ssm::StepParams p{};
  p.x_new = x_new; p.conv_state = conv_state; p.conv_weight = conv_weight;
  p.conv_bias = conv_bias; p.conv_width = conv_state ? conv_width : 0;
  p.delta = delta; p.delta_bias = delta_bias; p.A_log = A_log;
  p.B = B; p.C = C; p.D = D; p.z = z; p.state = state; p.y = y;
  p.batch = dims.batch; p.dim = dims.dim; p.dstate = int(dims.dstate);
  p.softplus = (flags & SSM_DELTA_SOFTPLUS) ? 1 : 0;
  p.write_zoh = (flags & SSM_WRITE_ZOH) ? 1 : 0;
  const bool vec = (dims.dstate % 4 == 0) && aligned(state, 16) &&
                   aligned(B, 4 * esz) && aligned(C, 4 * esz);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The bulk-copy kernel: N = 4, 8 or 16 with rows of B and C at least 16
  // bytes, channel runs of whole 16-byte chunks, every buffer 16-byte
  // aligned and a conv buffer of at most 8 samples.
  bool bulk = !(h->debug & ssm::kDebugStepPerThread) &&
              (dims.dstate == 4 || dims.dstate == 8 || dims.dstate == 16) &&
              dims.dstate * esz >= 16 && (dims.dim * esz) % 16 == 0;
  {
    const void *runs[] = {x_new, delta, z, B, C, y, state, conv_state};
    for (const void *q : runs)
      if (q && !aligned(q, 16)) bulk = false;
  }
  if (bulk) {
    const int rc = ensure_ctl(h, s);
    if (rc != SSM_OK) return rc;
    p.status = h->ctl;
    p.spin_limit = h->spin_limit;
    // counters run to 2^32 rows; with more columns or rows, fixed strides
    if ((dims.dim + 127) / 128 <= kMaxRowCounters && dims.batch < (1ll << 31))
      p.row_counter = reinterpret_cast<unsigned *>(h->ctl + kCtlRowCounters);
    const int n = int(dims.dstate);
    if (dtype == SSM_F32)
      return n == 4    ? launch_step_bulk<float, 4>(p, h->sm_count, s)
             : n == 8 ? launch_step_bulk<float, 8>(p, h->sm_count, s)
                      : launch_step_bulk<float, 16>(p, h->sm_count, s);
    return n == 4    ? launch_step_bulk<__nv_bfloat16, 4>(p, h->sm_count, s)
           : n == 8 ? launch_step_bulk<__nv_bfloat16, 8>(p, h->sm_count, s)
                    : launch_step_bulk<__nv_bfloat16, 16>(p, h->sm_count, s);
  }
  return dtype == SSM_F32
             ? launch_step<float>(p, vec, h->sm_count, s)
             : launch_step<__nv_bfloat16>(p, vec, h->sm_count, s);
}

int ssm_scan_create(ssm_scan_t *out, int device) {
  if (!out) return SSM_ERR_INVALID;
  *out = nullptr;
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (device < 0 || device >= count) return SSM_ERR_INVALID;
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor,
                             device) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor,
                             device) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) !=
          cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (major != 10 || minor != 0) return SSM_ERR_ARCH;
  ssm_scan_s *h = new (std::nothrow) ssm_scan_s();
  if (!h) return SSM_ERR_NOMEM;
  h->device = device;
  h->sm_count = sms;
  *out = h;
  return SSM_OK;
}

int ssm_scan_destroy(ssm_scan_t h) {
  if (!h) return SSM_OK;
  int rc = SSM_OK;
  if (h->ws || h->ctl || h->ckpt || h->det || h->bdyn) {
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(h->device);
    if (h->ws && cudaFree(h->ws) != cudaSuccess) rc = SSM_ERR_CUDA;
    if (h->ctl && cudaFree(h->ctl) != cudaSuccess) rc = SSM_ERR_CUDA;
    if (h->ckpt && cudaFree(h->ckpt) != cudaSuccess) rc = SSM_ERR_CUDA;
    if (h->det && cudaFree(h->det) != cudaSuccess) rc = SSM_ERR_CUDA;
    if (h->bdyn && cudaFree(h->bdyn) != cudaSuccess) rc = SSM_ERR_CUDA;
    cudaSetDevice(prev);
  }
  delete h;
  return rc;
}

int ssm_scan_set_variant(ssm_scan_t h, int variant, int segments) {
  if (!h) return SSM_ERR_INVALID;
  if (variant < SSM_VARIANT_AUTO || variant > SSM_VARIANT_CHUNKED)
    return SSM_ERR_INVALID;
  if (segments < 0) return SSM_ERR_INVALID;
  h->variant = variant;
  h->segments = segments;
  return SSM_OK;
}

int ssm_scan_set_debug(ssm_scan_t h, unsigned flags, unsigned spin_limit) {
  if (!h) return SSM_ERR_INVALID;
  h->debug = flags;
  h->spin_limit = spin_limit ? spin_limit : kDefaultSpinLimit;
  return SSM_OK;
}

int ssm_scan_set_time_blocks(ssm_scan_t h, int time_blocks) {
  if (!h) return SSM_ERR_INVALID;
  if (time_blocks != 0 && time_blocks != 1 && time_blocks != 2 &&
      time_blocks != 4 && time_blocks != 8)
    return SSM_ERR_INVALID;
  h->time_blocks = time_blocks;
  return SSM_OK;
}

int ssm_scan_last_variant(ssm_scan_t h, int *variant, int *segments) {
  if (!h) return SSM_ERR_INVALID;
  if (variant) *variant = h->last_variant;
  if (segments) *segments = h->last_segments;
  return SSM_OK;
}

int ssm_scan_sync_status(ssm_scan_t h, struct CUstream_st *stream) {
  if (!h) return SSM_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (!h->ctl) return SSM_OK;
  int status = 0;
  if (cudaMemcpy(&status, h->ctl, sizeof(int), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return SSM_ERR_CUDA;
  if (status != ssm::kStatusOk) {
    const int zero = 0;
    if (cudaMemcpy(h->ctl, &zero, sizeof(int), cudaMemcpyHostToDevice) !=
        cudaSuccess)
      return SSM_ERR_CUDA;
    return SSM_ERR_TIMEOUT;
  }
  return SSM_OK;
}

const char *ssm_scan_status_string(int status) {
  switch (status) {
    case SSM_OK: return "ok";
    case SSM_ERR_INVALID: return "invalid argument";
    case SSM_ERR_UNSUPPORTED: return "unsupported dtype, state size or shape";
    case SSM_ERR_ALIGN: return "misaligned pointer";
    case SSM_ERR_ARCH: return "device is not compute capability 10.0 (sm_100a)";
    case SSM_ERR_CUDA: return "CUDA runtime error";
    case SSM_ERR_TIMEOUT: return "bounded wait between thread blocks timed out";
    case SSM_ERR_NOMEM: return "allocation failed";
    default: return "unknown status";
  }
}

int ssm_scan_fwd(ssm_scan_t h, const void *x, const void *delta,
                 const float *A_log, const void *B, const void *C,
                 const float *D, const void *z, const float *delta_bias,
                 uint32_t flags, const float *h0, void *y, float *h_last,
                 ssm_scan_dims dims, int dtype, struct CUstream_st *stream) {
  return scan_fwd(h, x, nullptr, nullptr, 0, delta, A_log, B, C, D, z,
                  delta_bias, flags, h0, y, h_last, dims, dtype,
                  reinterpret_cast<cudaStream_t>(stream));
}

int ssm_scan_fwd_conv(ssm_scan_t h, const void *v, const float *conv_weight,
                      const float *conv_bias, int conv_width,
                      const void *delta, const float *A_log, const void *B,
                      const void *C, const float *D, const void *z,
                      const float *delta_bias, uint32_t flags,
                      const float *h0, void *y, float *h_last,
                      ssm_scan_dims dims, int dtype,
                      struct CUstream_st *stream) {
  if (!conv_weight) return SSM_ERR_INVALID;
  return scan_fwd(h, v, conv_weight, conv_bias, conv_width, delta, A_log, B,
                  C, D, z, delta_bias, flags, h0, y, h_last, dims, dtype,
                  reinterpret_cast<cudaStream_t>(stream));
}

int ssm_scan_bwd(ssm_scan_t h, const void *x, const void *delta,
                 const float *A_log, const void *B, const void *C,
                 const float *D, const void *z, const float *delta_bias,
                 uint32_t flags, const float *h0, const void *dy,
                 const float *dh_last, void *dx, void *ddelta, float *dA_log,
                 float *dB, float *dC, float *dD, void *dz,
                 float *ddelta_bias, float *dh0, ssm_scan_dims dims, int dtype,
                 struct CUstream_st *stream) {
  // ---- host-side validation: nothing touches the GPU before it passes
  if (!h || !x || !delta || !A_log || !B || !C || !dy || !dx || !ddelta ||
      !dA_log || !dB || !dC)
    return SSM_ERR_INVALID;
  if ((z && !dz) || (D && !dD) || (delta_bias && !ddelta_bias))
    return SSM_ERR_INVALID;
  if (dims.batch <= 0 || dims.seqlen <= 0 || dims.dim <= 0 || dims.dstate <= 0)
    return SSM_ERR_INVALID;
  if (flags & ~uint32_t(SSM_DELTA_SOFTPLUS | SSM_WRITE_ZOH |
                        SSM_REUSE_CHECKPOINTS | SSM_DETERMINISTIC))
    return SSM_ERR_INVALID;
  const bool reuse = (flags & SSM_REUSE_CHECKPOINTS) != 0;
  const bool det = (flags & SSM_DETERMINISTIC) != 0;
  flags &= ~uint32_t(SSM_REUSE_CHECKPOINTS | SSM_DETERMINISTIC);
  if (dtype != SSM_F32 && dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  const int64_t N = dims.dstate;
  const size_t esz = dtype == SSM_F32 ? 4 : 2;
  if (N != 4 && N != 8 && N != 16) return SSM_ERR_UNSUPPORTED;
  if (N * int64_t(esz) < 16 || (dims.dim * int64_t(esz)) % 16 != 0)
    return SSM_ERR_UNSUPPORTED;
  int64_t rows = 0, acts = 0, st = 0, nck = 0, ck = 0;
  if (!mul_ok(dims.batch, dims.seqlen, &rows) ||
      !mul_ok(rows, dims.dim, &acts) ||
      !mul_ok(dims.batch * dims.dim, N, &st) || acts > (int64_t(1) << 56))
    return SSM_ERR_INVALID;
  nck = (dims.seqlen + ssm::kCkptSteps - 1) / ssm::kCkptSteps;
  if (!mul_ok(st, nck, &ck) || ck > (int64_t(1) << 56)) return SSM_ERR_INVALID;
  const void *tiles_in[] = {x, delta, z, dy, B, C};
  for (const void *q : tiles_in)
    if (q && !aligned(q, 16)) return SSM_ERR_ALIGN;
  const void *acts_out[] = {dx, ddelta, dz};
  for (const void *q : acts_out)
    if (q && !aligned(q, esz)) return SSM_ERR_ALIGN;
  const float *f4[] = {h0, dh_last, dh0, A_log, dB, dC};
  for (const float *q : f4)
    if (q && !aligned(q, 16)) return SSM_ERR_ALIGN;
  const float *f1[] = {D, delta_bias, dA_log, dD, ddelta_bias};
  for (const float *q : f1)
    if (q && !aligned(q, 4)) return SSM_ERR_ALIGN;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (cur != h->device) return SSM_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // ---- checkpoints: the training forward's, or a workspace for our own
  if (reuse) {
    const ssm_scan_dims &k = h->ckpt_dims;
    if (!h->ckpt_saved || k.batch != dims.batch || k.seqlen != dims.seqlen ||
        k.dim != dims.dim || k.dstate != dims.dstate ||
        h->ckpt_dtype != dtype || h->ckpt_flags != flags)
      return SSM_ERR_INVALID;
  } else {
    const int rc = ensure_ckpt(h, size_t(ck) * sizeof(float), s);
    if (rc != SSM_OK) return rc;
    h->ckpt_saved = false;  // this call's forward overwrites them
  }
  // ---- deterministic sums: the partial slices (every element written by
  // exactly one block, so nothing is cleared); else the summed outputs are
  // cleared for the atomics
  size_t det_parts[5] = {0, 0, 0, 0, 0};  // float offsets: dB dC dA dD db
  if (det) {
    const int64_t G = (32 / (N / 4)) * kBwdWarps;  // channels per block
    const int64_t tiles = (dims.dim + G - 1) / G;
    int64_t bln = 0, slice = 0;
    if (!mul_ok(rows, N, &bln) || !mul_ok(bln, tiles, &slice))
      return SSM_ERR_INVALID;
    const size_t en = size_t(dims.dim) * N, be = size_t(dims.batch) *
                                                   dims.dim;
    det_parts[1] = size_t(slice);
    det_parts[2] = 2 * size_t(slice);
    det_parts[3] = det_parts[2] + size_t(dims.batch) * en;
    det_parts[4] = det_parts[3] + be;
    const size_t need = (det_parts[4] + be) * sizeof(float);
    if (need > h->det_bytes) {
      if (h->det) cudaFreeAsync(h->det, s);
      h->det = nullptr;
      h->det_bytes = 0;
      if (cudaMallocAsync(reinterpret_cast<void **>(&h->det), need, s) !=
          cudaSuccess) {
        cudaGetLastError();
        return SSM_ERR_NOMEM;
      }
      h->det_bytes = need;
    }
  }
  const size_t bcn = size_t(rows) * N * sizeof(float);
  if (!det && (cudaMemsetAsync(dB, 0, bcn, s) != cudaSuccess ||
      cudaMemsetAsync(dC, 0, bcn, s) != cudaSuccess ||
      cudaMemsetAsync(dA_log, 0, size_t(dims.dim) * N * sizeof(float), s) !=
          cudaSuccess ||
      (dD && cudaMemsetAsync(dD, 0, size_t(dims.dim) * sizeof(float), s) !=
                 cudaSuccess) ||
      (ddelta_bias &&
       cudaMemsetAsync(ddelta_bias, 0, size_t(dims.dim) * sizeof(float), s) !=
           cudaSuccess)))
    return SSM_ERR_CUDA;

  ssm::ScanParams fp{};
  fp.x = x; fp.delta = delta; fp.A_log = A_log; fp.B = B; fp.C = C;
  fp.D = D; fp.z = z; fp.delta_bias = delta_bias; fp.h0 = h0;
  fp.y = nullptr; fp.h_last = nullptr; fp.ckpt = h->ckpt;
  fp.batch = dims.batch; fp.seqlen = dims.seqlen; fp.dim = dims.dim;
  fp.dstate = int(N);
  fp.softplus = (flags & SSM_DELTA_SOFTPLUS) ? 1 : 0;
  fp.write_zoh = (flags & SSM_WRITE_ZOH) ? 1 : 0;
  fp.segments = 1;

  ssm::BwdParams bp{};
  bp.x = x; bp.delta = delta; bp.z = z; bp.dy = dy; bp.B = B; bp.C = C;
  bp.A_log = A_log; bp.D = D; bp.delta_bias = delta_bias; bp.h0 = h0;
  bp.dh_last = dh_last; bp.ckpt = h->ckpt;
  if (det) {
    bp.part_dB = h->det + det_parts[0];
    bp.part_dC = h->det + det_parts[1];
    bp.part_dA = h->det + det_parts[2];
    bp.part_dD = h->det + det_parts[3];
    bp.part_db = h->det + det_parts[4];
  }
  bp.dx = dx; bp.ddelta = ddelta; bp.dz = z ? dz : nullptr;
  bp.dB = dB; bp.dC = dC; bp.dA_log = dA_log;
  bp.dD = D ? dD : nullptr; bp.ddelta_bias = delta_bias ? ddelta_bias : nullptr;
  bp.dh0 = dh0;
  bp.batch = dims.batch; bp.seqlen = dims.seqlen; bp.dim = dims.dim;
  bp.dstate = int(N); bp.softplus = fp.softplus;

  if (dtype == SSM_BF16) {
    if (N == 16) return run_bwd<C16b1, __nv_bfloat16, 4>(h, fp, bp, reuse, s);
    return run_bwd<C8b1, __nv_bfloat16, 2>(h, fp, bp, reuse, s);
  }
  if (N == 16) return run_bwd<C16f1, float, 4>(h, fp, bp, reuse, s);
  if (N == 8) return run_bwd<C8f1, float, 2>(h, fp, bp, reuse, s);
  return run_bwd<C4f1, float, 1>(h, fp, bp, reuse, s);
}

}  // extern "C"
