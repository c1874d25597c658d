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
// consecutive channels and a contiguous range of steps; it walks that range in
// windows of TW steps. Inside a warp a lane is (c, g, q):
//   c: one of CW channels of the warp,
//   g: one of NG groups of 4 state coordinates (N = 4 NG),
//   q: one of TB time blocks: with TB > 1 the TB lanes of a (c, g) pair own
//      consecutive K-step blocks of a sub-window, fold their steps into one
//      affine map, combine the maps with a warp-shuffle scan and then replay
//      their steps from the true incoming state (time parallelism inside the
//      warp); with TB == 1 a lane walks every step itself.
// Each lane keeps its 4 states in float32 registers across windows; states of
// intermediate steps never leave the chip.
//
// Per window: x, raw delta, z tiles [TW x G] and B, C tiles [TW x N] are
// staged in shared memory with cp.async (double buffered, one window ahead;
// rows padded so the lane access patterns are bank-conflict free); bfloat16
// B and C are widened once per window to float32. For each block of NG steps
// the NG lanes of a (c, q) pair each compute softplus for one step (so every
// (t, e) pays its softplus once) and exchange (delta, delta*x) by shuffles.
// The readout partial sums over each lane's 4 states are combined over the NG
// lanes by a transposing butterfly that leaves lane g holding the full y of
// the block's step g, which then adds D x, applies the SiLU gate, and stores.
#pragma once

#include <float.h>

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
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
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
  static constexpr int BF_BYTES = round16(TW * BF_ROW + (TW / K) * BF_PB);
  static constexpr int BCRAW_BYTES = ESZ == 2 ? round16(TW * N * 2) : 0;
  static constexpr int STAGE_BYTES =
      3 * RAW_BYTES + (ESZ == 2 ? 2 * BCRAW_BYTES : 2 * BF_BYTES);
  static constexpr int SMEM_BYTES =
      2 * STAGE_BYTES + (ESZ == 2 ? 2 * BF_BYTES : 0);
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

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS)
scan_chunked_kernel(const ScanParams p) {
  using T = typename Cfg::T;
  constexpr int NG = Cfg::NG, TB = Cfg::TB, K = Cfg::K, TW = Cfg::TW;
  constexpr int CW = Cfg::CW, G = Cfg::G, N = Cfg::N, ESZ = Cfg::ESZ;
  constexpr int THREADS = Cfg::THREADS;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ __align__(16) unsigned char smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q = lane % TB;
  const int g = (lane / TB) % NG;
  const int c = lane / (TB * NG);
  const int cl = warp * CW + c;  // channel within the tile

  const int64_t L = p.seqlen, E = p.dim;
  const int64_t tiles = (E + G - 1) / G;
  const int64_t b = blockIdx.x / tiles;
  const int64_t e0 = (blockIdx.x - b * tiles) * G;
  const int64_t e = e0 + cl;
  const bool ch_ok = e < E;

  const T *gx = static_cast<const T *>(p.x);
  const T *gdl = static_cast<const T *>(p.delta);
  const T *gz = static_cast<const T *>(p.z);
  const T *gB = static_cast<const T *>(p.B);
  const T *gC = static_cast<const T *>(p.C);
  T *gy = static_cast<T *>(p.y);
  const bool has_z = gz != nullptr;

  float A2[4];     // A * log2(e) for this lane's 4 states
  float carry[4];  // state entering the next (sub-)window
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    A2[i] = 0.0f;
    carry[i] = 0.0f;
    if (ch_ok) {
      // clamp so that a zero step never meets -inf (0 * -inf = NaN)
      A2[i] = fmaxf(-expf(p.A_log[e * N + 4 * g + i]) * kLog2e, -FLT_MAX);
      if (p.h0) carry[i] = p.h0[(b * E + e) * N + 4 * g + i];
    }
  }
  const float bias = (ch_ok && p.delta_bias) ? p.delta_bias[e] : 0.0f;
  const float Dv = (ch_ok && p.D) ? p.D[e] : 0.0f;

  float *const bf_conv = reinterpret_cast<float *>(smem + 2 * Cfg::STAGE_BYTES);

  // ---- issue the copies of window w into stage s
  auto stage = [&](int64_t w, int s) {
    unsigned char *base = smem + s * Cfg::STAGE_BYTES;
    const int64_t t0 = w * TW;
    constexpr int CPR = Cfg::RAW_ROW / 16;  // 16-byte chunks per tile row
    constexpr int EPC = 16 / ESZ;           // elements per chunk
    for (int idx = tid; idx < TW * CPR; idx += THREADS) {
      const int r = idx / CPR, k = idx - (idx / CPR) * CPR;
      const int64_t t = t0 + r;
      const int64_t ec = e0 + k * EPC;
      const bool ok = t < L && ec < E;
      const int64_t go = ok ? (b * L + t) * E + ec : 0;
      const int so = Cfg::raw_off(r) + k * 16;
      cp_async16(base + so, gx + go, ok);
      cp_async16(base + Cfg::RAW_BYTES + so, gdl + go, ok);
      if (has_z) cp_async16(base + 2 * Cfg::RAW_BYTES + so, gz + go, ok);
    }
    unsigned char *bc = base + 3 * Cfg::RAW_BYTES;
    if constexpr (ESZ == 2) {
      // dense [TW][N] bfloat16 rows, contiguous in memory
      constexpr int CH = TW * N * 2 / 16;
      for (int idx = tid; idx < CH; idx += THREADS) {
        const int r = idx * 16 / (N * 2);
        const bool ok = t0 + r < L;
        const int64_t go = ok ? (b * L + t0) * N + (int64_t)idx * 8 : 0;
        cp_async16(bc + idx * 16, gB + go, ok);
        cp_async16(bc + Cfg::BCRAW_BYTES + idx * 16, gC + go, ok);
      }
    } else {
      // float rows of N*4 bytes straight into the padded float layout
      constexpr int CPRB = N * 4 / 16;
      for (int idx = tid; idx < TW * CPRB; idx += THREADS) {
        const int r = idx / CPRB, k = idx - (idx / CPRB) * CPRB;
        const bool ok = t0 + r < L;
        const int64_t go = ok ? (b * L + t0 + r) * N + k * 4 : 0;
        const int so = Cfg::bf_off(r) + k * 16;
        cp_async16(bc + so, gB + go, ok);
        cp_async16(bc + Cfg::BF_BYTES + so, gC + go, ok);
      }
    }
  };

  const int64_t nwin = (L + TW - 1) / TW;
  stage(0, 0);
  cp_async_commit();

  float h[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = carry[i];

  for (int64_t w = 0; w < nwin; ++w) {
    if (w + 1 < nwin) stage(w + 1, (w + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const unsigned char *base = smem + (w & 1) * Cfg::STAGE_BYTES;
    const unsigned char *sX = base;
    const unsigned char *sDL = base + Cfg::RAW_BYTES;
    const unsigned char *sZ = base + 2 * Cfg::RAW_BYTES;
    const float *sB;
    const float *sC;
    if constexpr (ESZ == 2) {
      const __nv_bfloat162 *rb = reinterpret_cast<const __nv_bfloat162 *>(
          base + 3 * Cfg::RAW_BYTES);
      const __nv_bfloat162 *rc = reinterpret_cast<const __nv_bfloat162 *>(
          base + 3 * Cfg::RAW_BYTES + Cfg::BCRAW_BYTES);
      float *fb = bf_conv;
      float *fc = reinterpret_cast<float *>(
          reinterpret_cast<unsigned char *>(bf_conv) + Cfg::BF_BYTES);
      for (int idx = tid; idx < TW * N / 2; idx += THREADS) {
        const int r = idx * 2 / N, n = idx * 2 - r * N;
        const int o = (Cfg::bf_off(r) >> 2) + n;
        const float2 vb = __bfloat1622float2(rb[idx]);
        const float2 vc = __bfloat1622float2(rc[idx]);
        *reinterpret_cast<float2 *>(fb + o) = vb;
        *reinterpret_cast<float2 *>(fc + o) = vc;
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

    // the raw (x, delta, z) of row r for this lane's channel
    auto load_raw = [&](int r, float &xv, float &dv, float &zv) {
      const int o = Cfg::raw_off(r) + cl * ESZ;
      xv = Act<T>::load(reinterpret_cast<const T *>(sX + o));
      dv = Act<T>::load(reinterpret_cast<const T *>(sDL + o));
      zv = has_z ? Act<T>::load(reinterpret_cast<const T *>(sZ + o)) : 0.0f;
    };
    // step size and step * x for row r (zero past the end of the sequence)
    auto step_of = [&](int r, float xv, float dv, float &dm, float &dxm) {
      const float v = dv + bias;
      dm = p.softplus ? softplus(v) : v;
      if (t0 + r >= L) dm = 0.0f;
      dxm = dm * xv;
    };
    auto finish = [&](int r, float yv, float xv, float zv) {
      yv = fmaf(Dv, xv, yv);
      if (has_z) yv *= silu(zv);
      const int64_t t = t0 + r;
      if (ch_ok && t < L) Act<T>::store(gy + (b * L + t) * E + e, yv);
    };

    if constexpr (TB == 1) {
#pragma unroll 2
      for (int jb = 0; jb < TW / NG; ++jb) {
        const int rm = jb * NG + g;
        float xm, dv, zm, dm, dxm;
        load_raw(rm, xm, dv, zm);
        step_of(rm, xm, dv, dm, dxm);
        float ps[NG];
#pragma unroll
        for (int s = 0; s < NG; ++s) {
          const int src = c * NG + s;
          const float ds = __shfl_sync(FULL, dm, src);
          const float dxs = __shfl_sync(FULL, dxm, src);
          const int r = jb * NG + s;
          const float4 Bq =
              *reinterpret_cast<const float4 *>(sB + (Cfg::bf_off(r) >> 2) + 4 * g);
          const float4 Cq =
              *reinterpret_cast<const float4 *>(sC + (Cfg::bf_off(r) >> 2) + 4 * g);
          const float bq[4] = {Bq.x, Bq.y, Bq.z, Bq.w};
          const float cq[4] = {Cq.x, Cq.y, Cq.z, Cq.w};
          float acc = 0.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a = ex2(ds * A2[i]);
            h[i] = fmaf(a, h[i], dxs * bq[i]);
            acc = fmaf(cq[i], h[i], acc);
          }
          ps[s] = acc;
        }
        const float yv = transpose_reduce<NG, TB>(ps, g);
        finish(rm, yv, xm, zm);
      }
    } else {
      constexpr int M = TW / Cfg::SUBWIN;
      constexpr int NB = K / NG;  // NG-step blocks per time block
#pragma unroll 1
      for (int m = 0; m < M; ++m) {
        const int r0 = m * Cfg::SUBWIN + q * K;  // first row of my time block
        float a[K][4], wr[K][4];
        float xs[NB], zs[NB];
        float Aa[4] = {1.0f, 1.0f, 1.0f, 1.0f};
        float Bb[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        // pass 1: per-step maps, folded into one map per time block
#pragma unroll
        for (int jb = 0; jb < NB; ++jb) {
          const int rm = r0 + jb * NG + g;
          float xm, dv, zm, dm, dxm;
          load_raw(rm, xm, dv, zm);
          step_of(rm, xm, dv, dm, dxm);
          xs[jb] = xm;
          zs[jb] = zm;
#pragma unroll
          for (int s = 0; s < NG; ++s) {
            const int src = (c * NG + s) * TB + q;
            const float ds = __shfl_sync(FULL, dm, src);
            const float dxs = __shfl_sync(FULL, dxm, src);
            const int j = jb * NG + s;
            const float4 Bq = *reinterpret_cast<const float4 *>(
                sB + (Cfg::bf_off(r0 + j) >> 2) + 4 * g);
            const float bq[4] = {Bq.x, Bq.y, Bq.z, Bq.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              a[j][i] = ex2(ds * A2[i]);
              wr[j][i] = dxs * bq[i];
              Bb[i] = fmaf(a[j][i], Bb[i], wr[j][i]);
              Aa[i] *= a[j][i];
            }
          }
        }
        // the incoming state enters at the first time block
        if (q == 0) {
#pragma unroll
          for (int i = 0; i < 4; ++i) Bb[i] = fmaf(Aa[i], carry[i], Bb[i]);
        }
        // inclusive warp-shuffle scan of the block maps over the TB lanes
#pragma unroll
        for (int d = 1; d < TB; d <<= 1) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float Ap = __shfl_up_sync(FULL, Aa[i], d, TB);
            const float Bp = __shfl_up_sync(FULL, Bb[i], d, TB);
            if (q >= d) {
              Bb[i] = fmaf(Aa[i], Bp, Bb[i]);
              Aa[i] *= Ap;
            }
          }
        }
        // Bb = state at the end of my block; the previous lane's is mine to
        // start from, the last lane's goes to the next sub-window
        float hs[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float prev = __shfl_up_sync(FULL, Bb[i], 1, TB);
          hs[i] = q == 0 ? carry[i] : prev;
          carry[i] = __shfl_sync(FULL, Bb[i], TB - 1, TB);
        }
        // pass 2: replay the block from the true incoming state, read out
#pragma unroll
        for (int jb = 0; jb < NB; ++jb) {
          float ps[NG];
#pragma unroll
          for (int s = 0; s < NG; ++s) {
            const int j = jb * NG + s;
            const float4 Cq = *reinterpret_cast<const float4 *>(
                sC + (Cfg::bf_off(r0 + j) >> 2) + 4 * g);
            const float cq[4] = {Cq.x, Cq.y, Cq.z, Cq.w};
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              hs[i] = fmaf(a[j][i], hs[i], wr[j][i]);
              acc = fmaf(cq[i], hs[i], acc);
            }
            ps[s] = acc;
          }
          const float yv = transpose_reduce<NG, TB>(ps, g);
          finish(r0 + jb * NG + g, yv, xs[jb], zs[jb]);
        }
      }
    }
    __syncthreads();
  }

  if (TB == 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) carry[i] = h[i];
  }
  if (p.h_last && ch_ok && q == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) p.h_last[(b * E + e) * N + 4 * g + i] = carry[i];
  }
}

}  // namespace ssm
