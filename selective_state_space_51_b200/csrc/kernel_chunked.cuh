// Chunked variant: the fused selective-scan forward for B200 (sm_100a).
//
// Recurrence (page "Mamba: Linear-Time Sequence Modeling with Selective State
// Spaces", www.abhik.ai/papers/mamba, section "Original paper, equations and
// runnable CPU code"): delta = softplus(raw + bias) [row 1];
// a = exp(delta A), A = -exp(A_log); h = a h + delta B x; y = sum_n C h + D x,
// read after the update [row 2]; y *= SiLU(z) [row 5]. Steps compose as affine
// maps (a2, w2) o (a1, w1) = (a2 a1, a2 w1 + w2) [row 3, and section "Compose
// the updates instead of waiting for every state"].
//
// Work decomposition. A thread block owns one batch row b, a tile of G
// consecutive channels and a contiguous piece of the sequence, walked in
// windows of TW steps. Inside a warp a lane is (c, g, q):
//   c: one of CW channels of the warp,
//   g: one of NG groups of 4 state coordinates (N = 4 NG),
//   q: one of TB time blocks. With TB > 1 the TB lanes of a (c, g) pair own
//      consecutive K-step blocks of each sub-window: each folds its steps into
//      one affine map, the maps are combined by a warp-shuffle scan, and each
//      lane then replays its steps from the true incoming state. With TB == 1
//      a lane walks every step itself.
// Each lane keeps its 4 states in float32 registers (two packed pairs, updated
// with FFMA2/FMUL2); states of intermediate steps never leave the chip.
//
// Per window: x, raw delta, z tiles [TW x G] and B, C tiles [TW x N] are
// staged in shared memory with cp.async (double buffered, one window ahead;
// rows padded so every lane access pattern is bank-conflict free); bfloat16
// B and C are widened to float32 once per window. With TB == 1 the steps go
// in blocks of 2 NG: lane g computes the step sizes of steps 2g and 2g+1
// (softplus on a packed pair) and publishes (delta, delta*x) for both in its
// channel's exchange row, so every (t, e) pays its softplus once; one block's
// step sizes are formed while the previous block's states are updated.
// Readout partials over each lane's 4 states are combined over the NG lanes
// by a transposing butterfly that leaves lane g the full y of steps 2g and
// 2g+1; lane g adds D x, applies the SiLU gate and stores. (With TB > 1 the
// blocks are NG steps, one per lane.) Options: the exact zero-order-hold
// write (ZOH), the causal convolution + SiLU that forms x from the staged
// input tile (CONV), and state checkpoints for the backward pass.
//
// Split sequences (SPLIT). For few channels and long sequences each sequence
// is cut into pieces scanned concurrently. A piece starts from a zero state,
// stores its outputs, and publishes its affine aggregate (end state from
// zero, product of retentions). It then looks back over its predecessors'
// publications (bounded waits) to learn its true incoming state, publishes
// its inclusive end state, and replays its first windows with no write term,
// adding C h * SiLU(z) to the stored outputs, until the carried-in part of the
// state has decayed to exactly zero (FTZ underflow). Blocks take pieces in
// launch-ticket order, so a block only ever waits for blocks already running.
#pragma once

#include <float.h>

#include <type_traits>

#include "device_math.cuh"
#include "scan_params.cuh"

namespace ssm {

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem,
                                           bool pred) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int src_size = pred ? 16 : 0;  // 0: fill the 16 bytes with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s),
               "l"(gmem), "r"(src_size)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void *smem, const void *gmem) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned *p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v)
               : "memory");
}

constexpr int round16(int x) { return (x + 15) / 16 * 16; }

// Tile geometry. RAW_PAD / RAW_PB / BF_PB are byte paddings (per row, and per
// block of BLK rows) chosen so that every lane access pattern of the kernel
// hits distinct banks (checked offline for each instantiated shape).
template <typename T_, int NG_, int TB_, int K_, int TW_, int NW_,
          int RAW_PAD_, int RAW_PB_, int BF_PB_>
struct ChunkCfg {
  using T = T_;
  static constexpr int NG = NG_, TB = TB_, K = K_, TW = TW_, NW = NW_;
  static constexpr int N = 4 * NG;
  static constexpr int CW = 32 / (NG * TB);
  static constexpr int G = CW * NW;
  static constexpr int THREADS = 32 * NW;
  static constexpr int ESZ = sizeof(T);
  static constexpr int BLK = TB > 1 ? K : NG;
  static constexpr int RAW_ROW = G * ESZ;
  static constexpr int RAW_P = RAW_ROW + RAW_PAD_;
  static constexpr int RAW_PB = RAW_PB_;
  static constexpr int RAW_BYTES = round16(TW * RAW_P + (TW / BLK) * RAW_PB);
  static constexpr int BF_ROW = N * 4;
  static constexpr int BF_PB = TB > 1 ? BF_PB_ : 0;
  static constexpr int BF_BYTES =
      round16(TW * BF_ROW + (TB > 1 ? (TW / K) * BF_PB : 0));
  static constexpr int BCRAW_BYTES = ESZ == 2 ? round16(TW * N * 2) : 0;
  static constexpr int STAGE_BYTES =
      3 * RAW_BYTES + (ESZ == 2 ? 2 * BCRAW_BYTES : 2 * BF_BYTES);
  // time-block-1 blocks: BS = 2 NG steps, 2 per lane; exchange rows of the
  // (delta, delta * x) pairs of a block, one row of BS pairs per channel.
  // Channels whose bit XRB is set keep their row's halves swapped (pair s at
  // s ^ BS/2), which makes both the 16-byte stores (8 lanes: 2 channels x 4
  // groups at N = 16) and the 16-byte loads of two steps' pairs free of bank
  // conflicts.
  static constexpr int BS = 2 * NG;
  static constexpr int SLOT = BS;
  static constexpr int XRB = NG == 4 ? 1 : 2;
  // per warp, 2 parities of: CW rows of SLOT pairs (time blocks 1) or 32
  // single slots (time blocks > 1)
  static constexpr int XCH_PER_WARP = TB == 1 ? CW * SLOT : 32;
  static constexpr int XCH_BYTES = NW * 2 * XCH_PER_WARP * 8;
  static constexpr int SMEM_BYTES =
      2 * STAGE_BYTES + (ESZ == 2 ? 2 * BF_BYTES : 0) + XCH_BYTES;
  static constexpr int SUBWIN = TB * K;  // steps per sub-window (TB > 1)

  static_assert(NG == 1 || NG == 2 || NG == 4, "N must be 4, 8 or 16");
  static_assert(32 % (NG * TB) == 0, "lane layout");
  static_assert(RAW_ROW % 16 == 0, "a tile row must be whole 16-byte chunks");
  static_assert(N * ESZ >= 16, "a B/C row must be at least one 16-byte chunk");
  static_assert(TB == 1 || TW % (TB * K) == 0, "window = sub-windows");
  static_assert(TB > 1 || TW % NG == 0, "window = blocks of NG steps");
  static_assert(K % NG == 0, "a time block holds whole NG-step blocks");
  static_assert(RAW_P % 16 == 0 && RAW_PB % 16 == 0 && BF_PB % 16 == 0,
                "cp.async destinations are 16-byte aligned");
  static_assert(TB > 1 || NG == 1 || (NG % 2 == 0 && SLOT * 8 % 16 == 0),
                "a half row of exchange pairs is whole 16-byte units");
  static_assert((TB > 1 ? K / NG : TW / (2 * NG)) % 2 == 0,
                "exchange slots alternate parity from block to block");
  static_assert(TW % kCkptSteps == 0 && kCkptSteps % (2 * NG) == 0,
                "checkpoints fall on block starts");

  __device__ static __forceinline__ int raw_off(int r) {
    return r * RAW_P + (r / BLK) * RAW_PB;
  }
  __device__ static __forceinline__ int bf_off(int r) {
    return r * BF_ROW + (TB > 1 ? (r / K) * BF_PB : 0);
  }
};

// Sum of p[s] over the NG lanes of a (c, q) pair, transposed: lane g ends up
// with the total of step s = g. Lane bits of g sit above the TB bits.
template <int NG, int TB>
__device__ __forceinline__ float transpose_reduce(const float (&p)[NG], int g) {
  constexpr unsigned FULL = 0xffffffffu;
  if constexpr (NG == 1) {
    return p[0];
  } else if constexpr (NG == 2) {
    const bool lo = g & 1;
    const float send = lo ? p[0] : p[1];
    const float keep = lo ? p[1] : p[0];
    return keep + __shfl_xor_sync(FULL, send, TB);
  } else {
    const bool hi = g & 2;
    const float s0 = hi ? p[0] : p[2], s1 = hi ? p[1] : p[3];
    float k0 = hi ? p[2] : p[0], k1 = hi ? p[3] : p[1];
    k0 += __shfl_xor_sync(FULL, s0, 2 * TB);
    k1 += __shfl_xor_sync(FULL, s1, 2 * TB);
    const bool lo = g & 1;
    const float s = lo ? k0 : k1;
    const float k = lo ? k1 : k0;
    return k + __shfl_xor_sync(FULL, s, TB);
  }
}

// Sum over the NG lanes of a (c, q) pair of 2 NG per-step partials, leaving
// lane g the totals of steps 2g and 2g+1 (a pair).
template <int NG, int TB>
__device__ __forceinline__ float2 transpose_reduce2(const float (&p)[2 * NG],
                                                    int g) {
  constexpr unsigned FULL = 0xffffffffu;
  auto shfl2 = [](float2 v, int m) {
    return make_float2(__shfl_xor_sync(FULL, v.x, m),
                       __shfl_xor_sync(FULL, v.y, m));
  };
  if constexpr (NG == 1) {
    return make_float2(p[0], p[1]);
  } else if constexpr (NG == 2) {
    const float2 P0 = make_float2(p[0], p[1]), P1 = make_float2(p[2], p[3]);
    const bool lo = g & 1;
    return add2(lo ? P1 : P0, shfl2(lo ? P0 : P1, TB));
  } else {
    const float2 P0 = make_float2(p[0], p[1]), P1 = make_float2(p[2], p[3]);
    const float2 P2 = make_float2(p[4], p[5]), P3 = make_float2(p[6], p[7]);
    const bool hi = g & 2;
    const float2 k0 = add2(hi ? P2 : P0, shfl2(hi ? P0 : P2, 2 * TB));
    const float2 k1 = add2(hi ? P3 : P1, shfl2(hi ? P1 : P3, 2 * TB));
    const bool lo = g & 1;
    return add2(lo ? k1 : k0, shfl2(lo ? k0 : k1, TB));
  }
}

enum { kWalkMain = 0, kWalkCorrect = 1 };

// FAST: the launch guarantees whole channel tiles (E a multiple of G), whole
// windows (L a multiple of TW), a gate, the softplus step and no checkpoints,
// so none of those is tested at run time (with or without the fused
// convolution).
// CKPT: the training forward of the backward pass. It writes the state
// before every kCkptSteps-th step and nothing else: no readout, no gate, no
// y, so C and z are neither staged nor read. With FAST it also needs only
// whole tiles and windows and the softplus step.
// SAVE: the specialised path's forward that also writes those checkpoints
// (y and all), for a backward that reuses them.
template <class Cfg, bool SPLIT, bool ZOH = false, bool CONV = false,
          bool FAST = false, bool CKPT = false, bool SAVE = false,
          bool DYN = false>
__global__ void __launch_bounds__(Cfg::THREADS)
scan_chunked_kernel(const ScanParams p) {
  static_assert(!ZOH || Cfg::TB == 1,
                "the zero-order-hold write runs with one time block");
  static_assert(!FAST || (Cfg::TB == 1 && !SPLIT && !ZOH),
                "the specialised path is the one-time-block, unsplit scan");
  static_assert(!CONV || Cfg::TB == 1,
                "the fused convolution runs with one time block");
  static_assert(!CKPT || (Cfg::TB == 1 && !SPLIT && !CONV),
                "checkpoints are written by the unsplit one-time-block scan");
  static_assert(!SAVE || (FAST && !CKPT && !CONV),
                "SAVE is the specialised forward that keeps its checkpoints");
  static_assert(!DYN || (FAST && !SPLIT),
                "DYN is the specialised scan run by persistent blocks");
  using T = typename Cfg::T;
  constexpr int NG = Cfg::NG, TB = Cfg::TB, K = Cfg::K, TW = Cfg::TW;
  constexpr int CW = Cfg::CW, G = Cfg::G, N = Cfg::N, ESZ = Cfg::ESZ;
  constexpr int THREADS = Cfg::THREADS;
  constexpr unsigned FULL = 0xffffffffu;
  // the specialised bfloat16 scan stages B and C interleaved per state group
  // (with the fused convolution this measured slower, so that keeps them
  // apart)
  constexpr bool BC_PAIRED = ESZ == 2 && FAST && !CKPT && !CONV;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ unsigned s_word;
  // fused convolution: the last KH inputs of the previous window, per channel
  // of the tile, for each window parity
  constexpr int KH = kScanConvMaxWidth - 1;
  __shared__ float s_halo[CONV ? 2 * KH * G : 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q = lane % TB;
  const int g = (lane / TB) % NG;
  const int c = lane / (TB * NG);
  const int cl = warp * CW + c;  // channel within the tile

  const int64_t L = p.seqlen, E = p.dim;
  const int64_t tiles = (E + G - 1) / G;

  // DYN: the blocks are persistent workers, as many as leave every
  // scheduler the same number of warps. Each pass takes the next unit (a
  // chunk of seg_len steps of one batch row and channel tile) in ticket
  // order, chunks of all tiles before the next chunk of any, waits until
  // the previous chunk of its tile has published its end state, starts
  // from that state and publishes its own. The state carried is exact, so
  // no chunk is replayed, and the load stays even at chunk granularity.
  for (;;) {
  // ---- which (piece, batch row, channel tile) this block scans
  int64_t unit = blockIdx.x;
  if constexpr (SPLIT || DYN) {
    if (tid == 0) s_word = atomicAdd(p.ticket, 1u);
    __syncthreads();
    unit = s_word;
    __syncthreads();
  }
  if constexpr (DYN)
    if (unit >= int64_t(p.segments) * p.batch * tiles) break;
  const int64_t seg = unit / (p.batch * tiles);
  const int64_t rem = unit - seg * p.batch * tiles;
  const int64_t b = rem / tiles;
  const int64_t tile = rem - b * tiles;
  const int64_t e0 = tile * G;
  const int64_t e = e0 + cl;
  const bool ch_ok = FAST || e < E;
  const int64_t t_begin = (SPLIT || DYN) ? seg * p.seg_len : 0;
  const int64_t t_end = (SPLIT || DYN) ? min(L, t_begin + p.seg_len) : L;

  const T *gx = static_cast<const T *>(p.x);
  const T *gdl = static_cast<const T *>(p.delta);
  const T *gz = static_cast<const T *>(p.z);
  const T *gB = static_cast<const T *>(p.B);
  const T *gC = static_cast<const T *>(p.C);
  T *gy = static_cast<T *>(p.y);
  const bool has_z = !CKPT && (FAST || gz != nullptr);
  const bool store_y = !CKPT && (FAST || gy != nullptr);
  const bool use_softplus = FAST || p.softplus;

  float2 A01 = make_float2(0.0f, 0.0f), A23 = A01;  // A * log2(e)
  float2 iA01 = A01, iA23 = A01;  // 1 / A (zero-order-hold write only)
  float2 h01 = A01, h23 = A01;  // state (TB == 1) or carry (TB > 1)
  if (ch_ok) {
    const float *al = p.A_log + e * N + 4 * g;
    if constexpr (ZOH) {
      iA01 = make_float2(-expf(-al[0]), -expf(-al[1]));
      iA23 = make_float2(-expf(-al[2]), -expf(-al[3]));
    }
    // clamp so that a zero step never meets -inf (0 * -inf = NaN)
    A01 = make_float2(fmaxf(-expf(al[0]) * kLog2e, -FLT_MAX),
                      fmaxf(-expf(al[1]) * kLog2e, -FLT_MAX));
    A23 = make_float2(fmaxf(-expf(al[2]) * kLog2e, -FLT_MAX),
                      fmaxf(-expf(al[3]) * kLog2e, -FLT_MAX));
    if (p.h0 && seg == 0) {
      const float *hp = p.h0 + (b * E + e) * N + 4 * g;
      h01 = make_float2(hp[0], hp[1]);
      h23 = make_float2(hp[2], hp[3]);
    }
  }
  if constexpr (DYN) {
    if (seg > 0) {
      // the previous chunk's end state, once it is published (bounded wait;
      // on timeout the status word says so and the chunk starts from zero)
      const unsigned *flag =
          p.flags + (b * p.segments + seg - 1) * tiles + tile;
      if (tid == 0) {
        const unsigned want = (p.epoch << 2) | kFlagInclusive;
        bool ok = false;
        for (unsigned spin = 0; spin < p.spin_limit; ++spin) {
          if (ld_acquire(flag) == want) {
            ok = true;
            break;
          }
          __nanosleep(64);
        }
        s_word = ok ? 1u : 0u;
        if (!ok) atomicExch(p.status, kStatusTimeout);
      }
      __syncthreads();
      const bool got = s_word != 0;
      __syncthreads();
      float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (got)
        v = __ldcg(reinterpret_cast<const float4 *>(
            p.incl_state + ((b * p.segments + seg - 1) * E + e) * N + 4 * g));
      h01 = make_float2(v.x, v.y);
      h23 = make_float2(v.z, v.w);
    }
  }
  const float bias = (ch_ok && p.delta_bias) ? p.delta_bias[e] : 0.0f;
  const float Dv = (ch_ok && p.D) ? p.D[e] : 0.0f;
  // float32: step sizes below this keep all four retentions on the
  // near-1 polynomial
  const float near_bound = near1_bound(A01, A23);
  (void)near_bound;
  // fused convolution weights, right-aligned: cw[kScanConvMaxWidth - 1]
  // multiplies the newest input, leading taps of a narrower filter are zero
  float cw[kScanConvMaxWidth] = {};
  float cbias = 0.0f;
  if constexpr (CONV) {
    if (ch_ok) {
      const int Kw = p.conv_width;
#pragma unroll
      for (int k = 0; k < kScanConvMaxWidth; ++k) {
        const int kk = k - (kScanConvMaxWidth - Kw);
        cw[k] = kk >= 0 ? p.conv_weight[e * Kw + kk] : 0.0f;
      }
      cbias = p.conv_bias ? p.conv_bias[e] : 0.0f;
    }
  }
  float2 P01 = make_float2(1.0f, 1.0f), P23 = P01;  // product of retentions

  float *const bf_conv = reinterpret_cast<float *>(smem + 2 * Cfg::STAGE_BYTES);
  float2 *const xch = reinterpret_cast<float2 *>(
      smem + 2 * Cfg::STAGE_BYTES + (ESZ == 2 ? 2 * Cfg::BF_BYTES : 0)) +
      warp * 2 * Cfg::XCH_PER_WARP;

  // ---- issue the copies of window w into stage s
  auto stage = [&](int64_t w, int s) {
    unsigned char *base = smem + s * Cfg::STAGE_BYTES;
    const int64_t t0 = w * TW;
    constexpr int CPR = Cfg::RAW_ROW / 16;  // 16-byte chunks per tile row
    constexpr int EPC = 16 / ESZ;           // elements per chunk
#pragma unroll
    for (int it = 0; it < (TW * CPR + THREADS - 1) / THREADS; ++it) {
      const int idx = tid + it * THREADS;
      if ((TW * CPR) % THREADS != 0 && idx >= TW * CPR) break;
      const int r = idx / CPR, k = idx - (idx / CPR) * CPR;
      const int64_t t = t0 + r;
      const int64_t ec = e0 + k * EPC;
      const bool ok = FAST || (t < t_end && ec < E);
      const int64_t go = ok ? (b * L + t) * E + ec : 0;
      const int so = Cfg::raw_off(r) + k * 16;
      cp_async16(base + so, gx + go, ok);
      cp_async16(base + Cfg::RAW_BYTES + so, gdl + go, ok);
      if (has_z) cp_async16(base + 2 * Cfg::RAW_BYTES + so, gz + go, ok);
    }
    unsigned char *bc = base + 3 * Cfg::RAW_BYTES;
    if constexpr (BC_PAIRED) {
      // the specialised path's B and C interleaved per state group: 16-byte
      // unit (r, g) holds B[r, 4g .. 4g+3] then C[r, 4g .. 4g+3], so a lane
      // reads both with one 16-byte load
      constexpr int U = TW * N / 4;  // 8-byte units per matrix
#pragma unroll
      for (int it = 0; it < (2 * U + THREADS - 1) / THREADS; ++it) {
        const int idx = tid + it * THREADS;
        if ((2 * U) % THREADS != 0 && idx >= 2 * U) break;
        const int q = idx >> 1, m = idx & 1;
        cp_async8(bc + q * 16 + m * 8,
                  (m ? gC : gB) + (b * L + t0) * N + int64_t(q) * 4);
      }
    } else if constexpr (ESZ == 2) {
      // dense [TW][N] bfloat16 rows, contiguous in memory
      constexpr int CH = TW * N * 2 / 16;
#pragma unroll
      for (int it = 0; it < (CH + THREADS - 1) / THREADS; ++it) {
        const int idx = tid + it * THREADS;
        if (CH % THREADS != 0 && idx >= CH) break;
        const int r = idx * 16 / (N * 2);
        const bool ok = FAST || t0 + r < t_end;
        const int64_t go = ok ? (b * L + t0) * N + (int64_t)idx * 8 : 0;
        cp_async16(bc + idx * 16, gB + go, ok);
        if constexpr (!CKPT)
          cp_async16(bc + Cfg::BCRAW_BYTES + idx * 16, gC + go, ok);
      }
    } else {
      // float rows of N*4 bytes straight into the padded float layout
      constexpr int CPRB = N * 4 / 16;
#pragma unroll
      for (int it = 0; it < (TW * CPRB + THREADS - 1) / THREADS; ++it) {
        const int idx = tid + it * THREADS;
        if ((TW * CPRB) % THREADS != 0 && idx >= TW * CPRB) break;
        const int r = idx / CPRB, k = idx - (idx / CPRB) * CPRB;
        const bool ok = FAST || t0 + r < t_end;
        const int64_t go = ok ? (b * L + t0 + r) * N + k * 4 : 0;
        const int so = Cfg::bf_off(r) + k * 16;
        cp_async16(bc + so, gB + go, ok);
        if constexpr (!CKPT) cp_async16(bc + Cfg::BF_BYTES + so, gC + go, ok);
      }
    }
  };

  // ---- walk windows [w_begin, w_end): MAIN stores y; CORRECT adds the
  // response of the carried-in state (no write term, no D x) to stored y and
  // stops as soon as that state is exactly zero everywhere in the block.
  auto walk = [&](auto mode_c, int64_t w_begin, int64_t w_end) {
    constexpr int MODE = decltype(mode_c)::value;
    stage(w_begin, 0);
    cp_async_commit();
    if constexpr (CONV) {
      if (MODE == kWalkMain) {
        // inputs just before the first window (zeros before the sequence)
        for (int idx = tid; idx < KH * G; idx += THREADS) {
          const int r = idx / G, ch = idx - (idx / G) * G;
          const int64_t t = w_begin * TW - KH + r;
          const int64_t ec = e0 + ch;
          s_halo[idx] = (t >= 0 && ec < E)
                            ? Act<T>::load(gx + (b * L + t) * E + ec)
                            : 0.0f;
        }
      }
    }
    for (int64_t w = w_begin; w < w_end; ++w) {
      const int par = int((w - w_begin) & 1);
      const int wpar = par;  // window parity (selects the halo)
      (void)wpar;
      if constexpr (FAST) {
        // this window's copies have landed and every thread is done with
        // the previous window's buffer: refill it with the next window
        cp_async_wait<0>();
        __syncthreads();
        if (w + 1 < w_end) stage(w + 1, par ^ 1);
        cp_async_commit();
      } else {
        if (w + 1 < w_end) stage(w + 1, par ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
      }

      const unsigned char *base = smem + par * Cfg::STAGE_BYTES;
      const unsigned char *sX = base;
      const unsigned char *sDL = base + Cfg::RAW_BYTES;
      const unsigned char *sZ = base + 2 * Cfg::RAW_BYTES;
      const float *sB = nullptr;
      const float *sC = nullptr;
      // bfloat16 B and C as staged (the specialised path reads them widened
      // in registers: B and C of a state group paired in one 16-byte load,
      // or, with the fused convolution, 8-byte loads of each; the others
      // from float copies)
      const T *const rawB =
          reinterpret_cast<const T *>(base + 3 * Cfg::RAW_BYTES);
      const T *const rawC = reinterpret_cast<const T *>(
          base + 3 * Cfg::RAW_BYTES + Cfg::BCRAW_BYTES);
      (void)rawB;
      (void)rawC;
      if constexpr (ESZ == 2 && FAST) {
      } else if constexpr (ESZ == 2) {
        const __nv_bfloat162 *rb = reinterpret_cast<const __nv_bfloat162 *>(
            base + 3 * Cfg::RAW_BYTES);
        const __nv_bfloat162 *rc = reinterpret_cast<const __nv_bfloat162 *>(
            base + 3 * Cfg::RAW_BYTES + Cfg::BCRAW_BYTES);
        float *fb = bf_conv;
        float *fc = reinterpret_cast<float *>(
            reinterpret_cast<unsigned char *>(bf_conv) + Cfg::BF_BYTES);
#pragma unroll
        for (int it = 0; it < (TW * N / 2 + THREADS - 1) / THREADS; ++it) {
          const int idx = tid + it * THREADS;
          if ((TW * N / 2) % THREADS != 0 && idx >= TW * N / 2) break;
          const int r = idx * 2 / N, n = idx * 2 - r * N;
          const int o = (Cfg::bf_off(r) >> 2) + n;
          *reinterpret_cast<float2 *>(fb + o) = __bfloat1622float2(rb[idx]);
          if constexpr (!CKPT)
            *reinterpret_cast<float2 *>(fc + o) = __bfloat1622float2(rc[idx]);
        }
        __syncthreads();
        sB = fb;
        sC = fc;
      } else {
        sB = reinterpret_cast<const float *>(base + 3 * Cfg::RAW_BYTES);
        sC = reinterpret_cast<const float *>(base + 3 * Cfg::RAW_BYTES +
                                             Cfg::BF_BYTES);
      }
      const int64_t t0 = w * TW;
      const int64_t ybase = (b * L + t0) * E + e;

      // this lane's step of a block: load its inputs, compute its step size,
      // publish (d, d, d x, d x) for the lanes of its channel and time block
      auto produce = [&](int r, int slot_par, float &xm, float &zm) {
        const int o = Cfg::raw_off(r) + cl * ESZ;
        xm = Act<T>::load(reinterpret_cast<const T *>(sX + o));
        const float dv = Act<T>::load(reinterpret_cast<const T *>(sDL + o));
        zm = has_z ? Act<T>::load(reinterpret_cast<const T *>(sZ + o)) : 0.0f;
        const float v = dv + bias;
        float dm = use_softplus ? softplus(v) : v;
        if (t0 + r >= t_end) dm = 0.0f;
        const float dxm = MODE == kWalkMain ? dm * xm : 0.0f;
        xch[slot_par * 32 + (c * TB + q) * NG + g] = make_float2(dm, dxm);
      };
      auto finish = [&](int r, float yv, float xm, float zm) {
        const int64_t t = t0 + r;
        if (MODE == kWalkMain) yv = fmaf(Dv, xm, yv);
        if (has_z) yv *= silu(zm);
        if (ch_ok && store_y && t < t_end) {
          T *yp = gy + ybase + int64_t(r) * E;
          if (MODE == kWalkCorrect) yv += Act<T>::load(yp);
          Act<T>::store(yp, yv);
        }
      };
      // one step of the 4 states: a = 2^(d A'), h = a h + d x B, partial C.h
      // B alone (the checkpointing forward reads no C)
      auto b_row = [&](int r, float4 &Bq) {
        if constexpr (ESZ == 2 && FAST) {
          Bq = Act<T>::load4(rawB + r * N + 4 * g);
        } else {
          Bq = *reinterpret_cast<const float4 *>(sB + (Cfg::bf_off(r) >> 2) +
                                                 4 * g);
        }
      };
      (void)b_row;
      auto bc_row = [&](int r, float4 &Bq, float4 &Cq) {
        if constexpr (BC_PAIRED) {
          const uint4 v = *reinterpret_cast<const uint4 *>(
              reinterpret_cast<const unsigned char *>(rawB) +
              (r * (N / 4) + g) * 16);
          Bq = make_float4(__uint_as_float(v.x << 16),
                           __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16),
                           __uint_as_float(v.y & 0xffff0000u));
          Cq = make_float4(__uint_as_float(v.z << 16),
                           __uint_as_float(v.z & 0xffff0000u),
                           __uint_as_float(v.w << 16),
                           __uint_as_float(v.w & 0xffff0000u));
        } else if constexpr (ESZ == 2 && FAST) {
          Bq = Act<T>::load4(rawB + r * N + 4 * g);
          Cq = Act<T>::load4(rawC + r * N + 4 * g);
        } else {
          const int o = (Cfg::bf_off(r) >> 2) + 4 * g;
          Bq = *reinterpret_cast<const float4 *>(sB + o);
          Cq = *reinterpret_cast<const float4 *>(sC + o);
        }
      };

      if constexpr (TB == 1) {
        // Blocks of BS = 2 NG steps. Lane g owns steps 2g and 2g+1 of a block:
        // it computes their step sizes (softplus on packed pairs) and
        // publishes them in its channel's exchange row, and after the
        // transposing reduction it finishes their outputs. Block jb's state
        // updates share an iteration with block jb+1's step sizes, so the two
        // dependency chains overlap. Exchange rows alternate parity; every
        // read of a row precedes the __syncwarp that ends its iteration.
        constexpr int BS = Cfg::BS, NBW = TW / BS, SLOT = Cfg::SLOT;
        (void)SLOT;
        // this channel's exchange row halves (see ChunkCfg::XRB)
        const int xswap = (c >> Cfg::XRB) & 1;
        const int xlo = c * SLOT + (xswap ? BS / 2 : 0);  // pairs 0 .. BS/2-1
        const int xhi = c * SLOT + (xswap ? 0 : BS / 2);  // pairs BS/2 ..
        const int xst = c * SLOT + ((2 * g) ^ (xswap ? BS / 2 : 0));
        (void)xlo;
        (void)xhi;
        (void)xst;
        // no step of the window is past the end
        const bool full = FAST || t0 + TW <= t_end;
        T *const yw = gy + ybase;

        // input of row r of the window; EDGE: r may be before the window
        auto vat = [&](int r, auto edge_c) -> float {
          if constexpr (decltype(edge_c)::value)
            if (r < 0) return s_halo[(wpar * KH + KH + r) * G + cl];
          return Act<T>::load(
              reinterpret_cast<const T *>(sX + Cfg::raw_off(r) + cl * ESZ));
        };
        auto produce2 = [&](int jb, int par, float2 &x2, float2 &z2,
                            float2 &dd0, float2 &dd1, auto edge_c) {
          const int r0 = jb * BS + 2 * g;
          const int o0 = Cfg::raw_off(r0) + cl * ESZ;
          const int o1 = Cfg::raw_off(r0 + 1) + cl * ESZ;
          x2 = make_float2(Act<T>::load(reinterpret_cast<const T *>(sX + o0)),
                           Act<T>::load(reinterpret_cast<const T *>(sX + o1)));
          if constexpr (CONV) {
            if (MODE == kWalkMain) {
              // x(r) = SiLU(bias + sum_k cw[k] v(r - 3 + k)), rows r0, r0+1
              const float vm3 = vat(r0 - 3, edge_c), vm2 = vat(r0 - 2, edge_c);
              const float vm1 = vat(r0 - 1, edge_c);
              float2 acc = make_float2(cbias, cbias);
              acc = fma2(make_float2(cw[0], cw[0]), make_float2(vm3, vm2), acc);
              acc = fma2(make_float2(cw[1], cw[1]), make_float2(vm2, vm1), acc);
              acc = fma2(make_float2(cw[2], cw[2]), make_float2(vm1, x2.x), acc);
              acc = fma2(make_float2(cw[3], cw[3]), x2, acc);
              x2 = PairMath<T>::silu(acc);
            }
          }
          const float2 v2 = add2(
              make_float2(Act<T>::load(reinterpret_cast<const T *>(sDL + o0)),
                          Act<T>::load(reinterpret_cast<const T *>(sDL + o1))),
              make_float2(bias, bias));
          z2 = has_z ? make_float2(
                           Act<T>::load(reinterpret_cast<const T *>(sZ + o0)),
                           Act<T>::load(reinterpret_cast<const T *>(sZ + o1)))
                     : make_float2(0.0f, 0.0f);
          float2 d2 = use_softplus ? PairMath<T>::softplus(v2) : v2;
          if (!full) {
            if (t0 + r0 >= t_end) d2.x = 0.0f;
            if (t0 + r0 + 1 >= t_end) d2.y = 0.0f;
          }
          // the second member is d x, or x itself for the zero-order-hold
          // write (its factor depends on the state)
          const float2 dx2 = MODE != kWalkMain ? make_float2(0.0f, 0.0f)
                             : ZOH          ? x2
                                            : mul2(d2, x2);
          dd0 = make_float2(d2.x, dx2.x);
          dd1 = make_float2(d2.y, dx2.y);
          if constexpr (NG > 1)
            *reinterpret_cast<float4 *>(xch + par * CW * SLOT + xst) =
                make_float4(d2.x, dx2.x, d2.y, dx2.y);
        };
        auto finish2 = [&](int jb, float2 y2, float2 x2, float2 z2) {
          const int r0 = jb * BS + 2 * g;
          if (MODE == kWalkMain) y2 = fma2(make_float2(Dv, Dv), x2, y2);
          if (has_z) y2 = mul2(y2, PairMath<T>::silu(z2));
          if (ch_ok && store_y) {
            T *yp = yw + int64_t(r0) * E;
            if (full || t0 + r0 < t_end) {
              if (MODE == kWalkCorrect) y2.x += Act<T>::load(yp);
              Act<T>::store(yp, y2.x);
            }
            if (full || t0 + r0 + 1 < t_end) {
              if (MODE == kWalkCorrect) y2.y += Act<T>::load(yp + E);
              Act<T>::store(yp + E, y2.y);
            }
          }
        };

        float2 x2, z2, e0, e1;
        produce2(0, 0, x2, z2, e0, e1, std::true_type());
        __syncwarp();
#pragma unroll 4
        for (int jb = 0; jb < NBW; ++jb) {
          const int par = jb & 1;
          if constexpr (!SPLIT && (!FAST || CKPT || SAVE)) {
            // training forward: the state before every kCkptSteps-th step
            if (MODE == kWalkMain && (CKPT || SAVE || p.ckpt) &&
                (jb * BS) % kCkptSteps == 0 && ch_ok &&
                t0 + jb * BS < t_end) {
              const int64_t k = (t0 + jb * BS) / kCkptSteps;
              const int64_t nck = (L + kCkptSteps - 1) / kCkptSteps;
              *reinterpret_cast<float4 *>(
                  p.ckpt + ((b * nck + k) * E + e) * N + 4 * g) =
                  make_float4(h01.x, h01.y, h23.x, h23.y);
            }
          }
          float2 dd[BS];
          if constexpr (NG > 1) {
            // two steps' pairs per 16-byte load (each half of the row is
            // whole 16-byte units: BS / 2 is even and rows start 16-byte
            // aligned)
#pragma unroll
            for (int s = 0; s < BS; s += 2) {
              const float4 v = *reinterpret_cast<const float4 *>(
                  xch + par * CW * SLOT +
                  (s < BS / 2 ? xlo + s : xhi + s - BS / 2));
              dd[s] = make_float2(v.x, v.y);
              dd[s + 1] = make_float2(v.z, v.w);
            }
          } else {
            dd[0] = e0;
            dd[1] = e1;
          }
          float2 xn = make_float2(0.f, 0.f), zn = xn, n0 = xn, n1 = xn;
          // a later block reaches before the window only with 2-step blocks
          if (jb + 1 < NBW)
            produce2(jb + 1, par ^ 1, xn, zn, n0, n1,
                     std::integral_constant<bool, (BS < KH)>());
          float ps[BS];
#pragma unroll
          for (int s = 0; s < BS; ++s) {
            float4 Bq, Cq;
            if constexpr (CKPT)
              b_row(jb * BS + s, Bq);
            else
              bc_row(jb * BS + s, Bq, Cq);
            const float2 dA = make_float2(dd[s].x, dd[s].x);
            const float2 zl01 = mul2(dA, A01), zl23 = mul2(dA, A23);
            float2 a01 = ex2x2(zl01);
            float2 a23 = ex2x2(zl23);
            if constexpr (ESZ == 4)  // float32: retentions near 1 exactly
              near1_retentions_warp(dd[s].x, near_bound, zl01, zl23, a01,
                                    a23);
            if (MODE == kWalkMain) {
              const float2 dx = make_float2(dd[s].y, dd[s].y);
              float2 w01 = mul2(dx, make_float2(Bq.x, Bq.y));
              float2 w23 = mul2(dx, make_float2(Bq.z, Bq.w));
              if constexpr (ZOH) {  // dx holds x: scale by expm1(dA)/A
                w01 = mul2(w01, zoh_factor2(dA, zl01, a01, iA01));
                w23 = mul2(w23, zoh_factor2(dA, zl23, a23, iA23));
              }
              h01 = fma2(a01, h01, w01);
              h23 = fma2(a23, h23, w23);
              if constexpr (SPLIT) {
                P01 = mul2(P01, a01);
                P23 = mul2(P23, a23);
              }
            } else {
              h01 = mul2(a01, h01);
              h23 = mul2(a23, h23);
            }
            if constexpr (!CKPT) {
              const float2 acc =
                  fma2(make_float2(Cq.z, Cq.w), h23,
                       mul2(make_float2(Cq.x, Cq.y), h01));
              ps[s] = acc.x + acc.y;
            }
          }
          if constexpr (!CKPT)
            finish2(jb, transpose_reduce2<NG, TB>(ps, g), x2, z2);
          x2 = xn;
          z2 = zn;
          e0 = n0;
          e1 = n1;
          __syncwarp();
        }
      } else {
        constexpr int M = TW / Cfg::SUBWIN;
        constexpr int NB = K / NG;  // NG-step blocks per time block
#pragma unroll 1
        for (int m = 0; m < M; ++m) {
          const int r0 = m * Cfg::SUBWIN + q * K;  // first row of my block
          float2 a01[K], a23[K], w01[K], w23[K];
          float xs[NB], zs[NB];
          float2 Aa01 = make_float2(1.0f, 1.0f), Aa23 = Aa01;
          float2 Bb01 = make_float2(0.0f, 0.0f), Bb23 = Bb01;
          // pass 1: per-step maps, folded into one map per time block
#pragma unroll
          for (int jb = 0; jb < NB; ++jb) {
            const int sp = jb & 1;
            produce(r0 + jb * NG + g, sp, xs[jb], zs[jb]);
            __syncwarp();
#pragma unroll
            for (int s = 0; s < NG; ++s) {
              const int j = jb * NG + s;
              const float2 dd = xch[sp * 32 + (c * TB + q) * NG + s];
              float4 Bq, Cq;
              bc_row(r0 + j, Bq, Cq);
              const float2 dA = make_float2(dd.x, dd.x);
              const float2 dx = make_float2(dd.y, dd.y);
              const float2 zl01 = mul2(dA, A01), zl23 = mul2(dA, A23);
              a01[j] = ex2x2(zl01);
              a23[j] = ex2x2(zl23);
              if constexpr (ESZ == 4)
                near1_retentions(dd.x, near_bound, zl01, zl23, a01[j],
                                 a23[j]);
              w01[j] = mul2(dx, make_float2(Bq.x, Bq.y));
              w23[j] = mul2(dx, make_float2(Bq.z, Bq.w));
              Bb01 = fma2(a01[j], Bb01, w01[j]);
              Bb23 = fma2(a23[j], Bb23, w23[j]);
              Aa01 = mul2(Aa01, a01[j]);
              Aa23 = mul2(Aa23, a23[j]);
            }
          }
          // the incoming state enters at the first time block
          if (q == 0) {
            Bb01 = fma2(Aa01, h01, Bb01);
            Bb23 = fma2(Aa23, h23, Bb23);
          }
          // inclusive warp-shuffle scan of the block maps over the TB lanes
#pragma unroll
          for (int d = 1; d < TB; d <<= 1) {
            float2 Ap01, Ap23, Bp01, Bp23;
            Ap01.x = __shfl_up_sync(FULL, Aa01.x, d, TB);
            Ap01.y = __shfl_up_sync(FULL, Aa01.y, d, TB);
            Ap23.x = __shfl_up_sync(FULL, Aa23.x, d, TB);
            Ap23.y = __shfl_up_sync(FULL, Aa23.y, d, TB);
            Bp01.x = __shfl_up_sync(FULL, Bb01.x, d, TB);
            Bp01.y = __shfl_up_sync(FULL, Bb01.y, d, TB);
            Bp23.x = __shfl_up_sync(FULL, Bb23.x, d, TB);
            Bp23.y = __shfl_up_sync(FULL, Bb23.y, d, TB);
            if (q >= d) {
              Bb01 = fma2(Aa01, Bp01, Bb01);
              Bb23 = fma2(Aa23, Bp23, Bb23);
              Aa01 = mul2(Aa01, Ap01);
              Aa23 = mul2(Aa23, Ap23);
            }
          }
          if constexpr (SPLIT) {
            if (MODE == kWalkMain) {
              // the whole sub-window's retention product sits in the last lane
              float2 S01, S23;
              S01.x = __shfl_sync(FULL, Aa01.x, TB - 1, TB);
              S01.y = __shfl_sync(FULL, Aa01.y, TB - 1, TB);
              S23.x = __shfl_sync(FULL, Aa23.x, TB - 1, TB);
              S23.y = __shfl_sync(FULL, Aa23.y, TB - 1, TB);
              P01 = mul2(P01, S01);
              P23 = mul2(P23, S23);
            }
          }
          // Bb = state at the end of my block. The previous lane's is mine to
          // start from; the last lane's carries to the next sub-window.
          float2 hs01, hs23;
          hs01.x = __shfl_up_sync(FULL, Bb01.x, 1, TB);
          hs01.y = __shfl_up_sync(FULL, Bb01.y, 1, TB);
          hs23.x = __shfl_up_sync(FULL, Bb23.x, 1, TB);
          hs23.y = __shfl_up_sync(FULL, Bb23.y, 1, TB);
          if (q == 0) {
            hs01 = h01;
            hs23 = h23;
          }
          h01.x = __shfl_sync(FULL, Bb01.x, TB - 1, TB);
          h01.y = __shfl_sync(FULL, Bb01.y, TB - 1, TB);
          h23.x = __shfl_sync(FULL, Bb23.x, TB - 1, TB);
          h23.y = __shfl_sync(FULL, Bb23.y, TB - 1, TB);
          // pass 2: replay the block from the true incoming state, read out
#pragma unroll
          for (int jb = 0; jb < NB; ++jb) {
            float ps[NG];
#pragma unroll
            for (int s = 0; s < NG; ++s) {
              const int j = jb * NG + s;
              float4 Bq, Cq;
              bc_row(r0 + j, Bq, Cq);
              hs01 = fma2(a01[j], hs01, w01[j]);
              hs23 = fma2(a23[j], hs23, w23[j]);
              const float2 acc =
                  fma2(make_float2(Cq.z, Cq.w), hs23,
                       mul2(make_float2(Cq.x, Cq.y), hs01));
              ps[s] = acc.x + acc.y;
            }
            finish(r0 + jb * NG + g, transpose_reduce<NG, TB>(ps, g), xs[jb],
                   zs[jb]);
          }
        }
      }
      if constexpr (CONV) {
        if (MODE == kWalkMain && w + 1 < w_end) {
          // the last KH inputs of this window open the next one
          for (int idx = tid; idx < KH * G; idx += THREADS) {
            const int r = idx / G, ch = idx - (idx / G) * G;
            s_halo[((wpar ^ 1) * KH + r) * G + ch] =
                Act<T>::load(reinterpret_cast<const T *>(
                    sX + Cfg::raw_off(TW - KH + r) + ch * ESZ));
          }
        }
      }
      if (MODE == kWalkCorrect) {
        const int alive = (h01.x != 0.0f) | (h01.y != 0.0f) |
                          (h23.x != 0.0f) | (h23.y != 0.0f);
        if (!__syncthreads_or(alive)) break;
      } else if constexpr (!FAST) {
        __syncthreads();
      }
    }
    cp_async_wait<0>();
    __syncthreads();
  };

  const int64_t w_begin = t_begin / TW;
  const int64_t w_end = (t_end + TW - 1) / TW;
  walk(std::integral_constant<int, kWalkMain>(), w_begin, w_end);

  float2 H01 = h01, H23 = h23;  // true end state of this piece
  if constexpr (DYN) {
    // (the publication test hook: the first chunk of each tile stays
    // unpublished, so its successor's bounded wait runs out)
    const bool suppress = (p.debug & kDebugNoPublish) && seg == 0;
    if (seg + 1 < p.segments && !suppress) {  // the next chunk starts here
      __stcg(reinterpret_cast<float4 *>(
                 p.incl_state + ((b * p.segments + seg) * E + e) * N + 4 * g),
             make_float4(h01.x, h01.y, h23.x, h23.y));
      __threadfence();
      __syncthreads();
      if (tid == 0)
        st_release(p.flags + (b * p.segments + seg) * tiles + tile,
                   (p.epoch << 2) | kFlagInclusive);
    }
  }
  if constexpr (SPLIT) {
    const int64_t S = p.segments;
    const int64_t slot = ((b * S + seg) * E + e) * N + 4 * g;
    unsigned *flag_of = p.flags + (b * S) * tiles + tile;  // + j * tiles
    const unsigned tag = p.epoch << 2;
    // publish the aggregate (the first piece's is already inclusive)
    if (ch_ok && q == 0) {
      if (seg == 0) {
        __stcg(reinterpret_cast<float4 *>(p.incl_state + slot),
               make_float4(h01.x, h01.y, h23.x, h23.y));
      } else {
        __stcg(reinterpret_cast<float4 *>(p.agg_state + slot),
               make_float4(h01.x, h01.y, h23.x, h23.y));
        __stcg(reinterpret_cast<float4 *>(p.agg_decay + slot),
               make_float4(P01.x, P01.y, P23.x, P23.y));
      }
    }
    __threadfence();
    __syncthreads();
    const bool suppress = (p.debug & kDebugNoPublish) && seg == 0;
    if (tid == 0 && !suppress)
      st_release(flag_of + seg * tiles,
                 tag | (seg == 0 ? kFlagInclusive : kFlagAggregate));

    if (seg > 0) {
      // look back: compose predecessors' aggregates until an inclusive one
      float2 cP01 = make_float2(1.0f, 1.0f), cP23 = cP01;  // map from there
      float2 cS01 = make_float2(0.0f, 0.0f), cS23 = cS01;  // to this start
      float2 hin01, hin23;
      for (int64_t j = seg - 1;; --j) {
        if (tid == 0) {
          unsigned f = 0, st = kFlagNone;
          for (unsigned spin = 0; spin < p.spin_limit; ++spin) {
            f = ld_acquire(flag_of + j * tiles);
            if ((f & ~3u) == tag && (f & 3u) != kFlagNone) {
              st = f & 3u;
              break;
            }
            __nanosleep(64);
          }
          s_word = st;
        }
        __syncthreads();
        const unsigned st = s_word;
        __syncthreads();
        const int64_t js = ((b * S + j) * E + e) * N + 4 * g;
        if (st == kFlagNone || j == 0 && st != kFlagInclusive) {
          if (tid == 0) atomicExch(p.status, kStatusTimeout);
          hin01 = cS01;
          hin23 = cS23;
          break;
        }
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (st == kFlagInclusive) {
          if (ch_ok) v = __ldcg(reinterpret_cast<const float4 *>(p.incl_state + js));
          hin01 = fma2(cP01, make_float2(v.x, v.y), cS01);
          hin23 = fma2(cP23, make_float2(v.z, v.w), cS23);
          break;
        }
        float4 u = v;
        if (ch_ok) {
          v = __ldcg(reinterpret_cast<const float4 *>(p.agg_state + js));
          u = __ldcg(reinterpret_cast<const float4 *>(p.agg_decay + js));
        }
        cS01 = fma2(cP01, make_float2(v.x, v.y), cS01);
        cS23 = fma2(cP23, make_float2(v.z, v.w), cS23);
        cP01 = mul2(cP01, make_float2(u.x, u.y));
        cP23 = mul2(cP23, make_float2(u.z, u.w));
      }
      // inclusive end state: own aggregate applied after the incoming state
      H01 = fma2(P01, hin01, h01);
      H23 = fma2(P23, hin23, h23);
      if (ch_ok && q == 0)
        __stcg(reinterpret_cast<float4 *>(p.incl_state + slot),
               make_float4(H01.x, H01.y, H23.x, H23.y));
      __threadfence();
      __syncthreads();
      if (tid == 0) st_release(flag_of + seg * tiles, tag | kFlagInclusive);
      // replay the start of the piece for the carried-in state's response
      h01 = hin01;
      h23 = hin23;
      if (!ch_ok) h01 = h23 = make_float2(0.0f, 0.0f);
      walk(std::integral_constant<int, kWalkCorrect>(), w_begin, w_end);
    }
  }

  if (p.h_last && ch_ok && q == 0 && t_end == L) {
    float *hp = p.h_last + (b * E + e) * N + 4 * g;
    hp[0] = H01.x;
    hp[1] = H01.y;
    hp[2] = H23.x;
    hp[3] = H23.y;
  }
  if constexpr (!DYN) break;
  }  // the DYN pass loop
}

}  // namespace ssm
