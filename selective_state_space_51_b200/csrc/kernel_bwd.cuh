// Backward pass of the selective scan: the reverse sweep.
//
// Page "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
// (www.abhik.ai/papers/mamba), section "Original paper, equations and
// runnable CPU code", rows 1, 2 and 5 define the forward recurrence; section
// "Compose the updates instead of waiting for every state" trains through it
// by recomputing states on the way back instead of storing them. With step
// size s, retention a_n = exp(s A_n), write w_n and the adjoint
// lam_n = d loss / d h_t[n], going backwards in time:
//   dy = g SiLU(z) (g = incoming gradient of the output), dz = g pre SiLU'(z)
//   with pre = C.h_t + D x;
//   lam += dy C;  dC[t, n] += dy h_t;  dD += dy x;  dx = dy D + sum lam f B;
//   ds = sum lam B x (f = s) or sum lam B x a (f = expm1(s A)/A)
//        + sum lam h_{t-1} a A;
//   dA += lam h_{t-1} a s  (+ lam B x (s a - f)/A for the zero-order hold);
//   dB[t, n] += lam f x;  lam <- lam a;  d raw = ds sigmoid(raw + bias).
//
// A thread block owns (batch row, G-channel tile) and the same (c, g) lanes
// as the forward kernel (NG lanes per channel, 4 states per lane). It walks
// windows of 16 steps from the last to the first. For each window:
//   1. the x, raw step, z, incoming-gradient, B and C tiles arrive by
//      cp.async (issued at the start of the previous window); B and C are
//      read from these staged tiles, in the activation type, throughout;
//   2. a pre-pass forms each (t, e)'s step size, x, dy, gate slope and
//      softplus slope once, in shared memory;
//   3. for each half window (one 8-step checkpoint interval), the later
//      half first, every lane recomputes its 4 states from the forward's
//      checkpoint at the start of that half, keeping them in shared memory;
//   4. the reverse sweep over the half updates lam in registers. The
//      per-channel sums (C.h, the dx and d-step partials) are buffered over
//      NG steps and summed over the channel's lanes by one transposing
//      butterfly.
// dB and dC are sums over channels. They stay off the sweep: before it, each
// warp sums dy h over its own channels straight from the state history; the
// sweep then overwrites each history slot, once no later step needs it, with
// the lane's lam f x, and a second warp pass sums those. Each pass ends in
// one 16-byte atomic add per lane into HBM.
#pragma once

#include "kernel_chunked.cuh"

namespace ssm {

struct BwdParams {
  const void *x, *delta, *z, *dy, *B, *C;  // activation dtype
  const float *A_log, *D, *delta_bias, *h0, *dh_last;
  const float *ckpt;  // [b, ceil(L / 8), E, N]: state before step 8 k
  // deterministic sums (DET): each block's share of the summed gradients,
  // added up afterwards in a fixed order instead of by atomics:
  // part_dB, part_dC [tiles][b, L, N]; part_dA [b][E, N]; part_dD, part_db
  // [b][E] (written only with D / delta_bias)
  float *part_dB, *part_dC, *part_dA, *part_dD, *part_db;
  // persistent blocks (DYN): units of (chunk, batch row, tile) taken from
  // *dyn_ticket; chunk k covers windows [nwin - (k + 1) W, nwin - k W)
  // (W = dyn_chunk_windows), chunks from the end of the sequence. A chunk
  // hands lam, the dA sums and the dD / bias partials of each thread to the
  // next (earlier) chunk through dyn_carry [b * tiles][threads][12] (10
  // used; rows 16-byte aligned), and
  // sets dyn_flags [b][dyn_chunks][tiles] (cleared before the launch).
  unsigned *dyn_ticket, *dyn_flags;
  float *dyn_carry;
  int dyn_chunks, dyn_chunk_windows;
  int *status;          // device status word (kStatusTimeout)
  unsigned spin_limit;  // polls of a hand-over wait
  unsigned debug;       // kDebugNoPublish: chunk 0 keeps its hand-over back
  void *dx, *ddelta, *dz;  // [b, L, E] activation dtype (dz: with z only)
  float *dB, *dC;          // [b, L, N], summed into (zero before the launch)
  float *dA_log;           // [E, N], summed into
  float *dD, *ddelta_bias;  // [E], summed into (with D / delta_bias only)
  float *dh0;              // [b, E, N] or nullptr
  int64_t batch, seqlen, dim;
  int dstate;
  int softplus;
};

template <typename T, int NG, int NW>
struct BwdCfg {
  static constexpr int N = 4 * NG, CW = 32 / NG, G = CW * NW;
  // windows of two checkpoint intervals; the state history of one interval
  // (half a window) is kept at a time
  static constexpr int THREADS = 32 * NW, TW = 2 * kCkptSteps;
  static constexpr int ESZ = sizeof(T);
  // raw tiles of one stage: x, raw step, z, dy [TW][G] and B, C [TW][N]
  static constexpr int ACT_BYTES = TW * G * ESZ;
  static constexpr int BC_BYTES = TW * N * ESZ;
  static constexpr int STAGE = 4 * ACT_BYTES + 2 * BC_BYTES;
  // per-window float arrays: s, x, dy, gate slope, softplus slope [TW][G];
  // the states of half a window [TW/2 + 1][RS] float4
  // row stride of the per-(t, e) arrays: the G channels plus 32 / NG words,
  // so that the NG lanes of a channel, which finish NG consecutive steps,
  // read distinct banks
  static constexpr int SP = G + (NG > 1 ? 32 / NG : 0);
  static constexpr int SCAL_BYTES = 5 * TW * SP * 4;
  static constexpr int HALF = kCkptSteps;  // rows of state history kept
  // history row stride in float4: 4 past THREADS, so that the two rows a
  // quarter-warp reads in the channel-sum passes fall on distinct banks.
  // Row 0 is the state before the half, row 1 + i the state after its
  // step i.
  static constexpr int RS = THREADS + 4;
  static constexpr int HIST_BYTES = (HALF + 1) * RS * 16;
  static constexpr int SMEM_BYTES = 2 * STAGE + SCAL_BYTES + HIST_BYTES;
  // lanes per (history row, quad of states) in the channel-sum passes: a
  // lane sums 8 channels of its warp
  static constexpr int K = 4 / NG;
  static_assert(HALF == 8 && CW == 8 * K,
                "channel-sum passes: 8 rows x 4 lanes per warp");
  static_assert(THREADS % G == 0, "a pre-pass thread keeps one channel pair");
  static_assert((G * ESZ) % 16 == 0 && (N * ESZ) % 16 == 0,
                "tile rows are whole 16-byte chunks");
};

// FAST: the launch guarantees whole channel tiles (E a multiple of G), whole
// windows (L a multiple of TW), a gate and the softplus step, so none of
// those is tested at run time.
// Held to 18 warps per SM (9 two-warp blocks: the shared-memory limit), so
// that the Mamba-2.8B layer's 1280 blocks are resident in one wave; the
// persistent variant to the 16 warps per SM it runs.
// DET: the summed gradients go to per-block partial slices (see BwdParams)
// instead of float32 atomics, so that a fixed-order reduction makes them
// bitwise reproducible; the NW warps of a block combine their channel sums
// through shared memory first, in warp order.
// DYN (with FAST): persistent blocks over (chunk, batch row, tile) units,
// the sweep's state handed from chunk to chunk (see BwdParams), so that
// every scheduler carries the same work where the tiles do not divide
// evenly over the SMs.
template <typename T, int NG, int NW, bool ZOH, bool FAST = false,
          bool DET = false, bool DYN = false>
__global__ void __launch_bounds__(32 * NW, (DYN ? 16 : 18) / NW)
    scan_bwd_kernel(const BwdParams p) {
  using Cfg = BwdCfg<T, NG, NW>;
  constexpr int N = Cfg::N, CW = Cfg::CW, G = Cfg::G, TW = Cfg::TW;
  constexpr int THREADS = Cfg::THREADS, ESZ = Cfg::ESZ, HALF = Cfg::HALF;
  constexpr int SP = Cfg::SP, RS = Cfg::RS, K = Cfg::K;
  constexpr unsigned FULL = 0xffffffffu;
  extern __shared__ __align__(16) unsigned char smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane % NG;
  const int c = lane / NG;
  const int cl = warp * CW + c;  // channel within the tile

  static_assert(!DYN || FAST, "persistent blocks run the specialised sweep");
  const int64_t L = p.seqlen, E = p.dim;
  const int64_t tiles = (E + G - 1) / G;
  const int64_t nwin = (L + TW - 1) / TW;
  const int64_t nck = (L + kCkptSteps - 1) / kCkptSteps;  // checkpoints
  __shared__ unsigned s_unit;
  (void)s_unit;

  for (;;) {  // DYN: one unit per pass; else one pass
  int64_t unit = blockIdx.x, chunk = 0;
  if constexpr (DYN) {
    if (tid == 0) s_unit = atomicAdd(p.dyn_ticket, 1u);
    __syncthreads();
    unit = s_unit;
    __syncthreads();
    if (unit >= int64_t(p.dyn_chunks) * p.batch * tiles) break;
    chunk = unit / (p.batch * tiles);
    unit -= chunk * p.batch * tiles;
  }
  const int64_t b = unit / tiles;
  const int64_t tile = unit - b * tiles;
  const int64_t e0 = tile * G;
  const int64_t e = e0 + cl;
  const bool ch_ok = FAST || e < E;
  // this unit's windows [w_lo, w_hi)
  const int64_t w_hi = DYN ? nwin - chunk * p.dyn_chunk_windows : nwin;
  const int64_t w_lo =
      DYN ? (w_hi > p.dyn_chunk_windows ? w_hi - p.dyn_chunk_windows : 0) : 0;

  float *const sS = reinterpret_cast<float *>(smem + 2 * Cfg::STAGE);
  float *const sX = sS + TW * SP;
  float *const sDY = sX + TW * SP;
  float *const sGZ = sDY + TW * SP;
  float *const sSG = sGZ + TW * SP;
  float4 *const sH = reinterpret_cast<float4 *>(sSG + TW * SP);

  const T *gx = static_cast<const T *>(p.x);
  const T *gdl = static_cast<const T *>(p.delta);
  const T *gz = static_cast<const T *>(p.z);
  const T *gdy = static_cast<const T *>(p.dy);
  const T *gB = static_cast<const T *>(p.B);
  const T *gC = static_cast<const T *>(p.C);
  const bool has_z = FAST || gz != nullptr;

  // per lane: A log2(e), 1/A, A for its 4 states
  float A2[4] = {}, iA[4] = {}, Av[4] = {};
  float lam[4] = {}, dA[4] = {};
  if (ch_ok) {
    const float *al = p.A_log + e * N + 4 * g;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      Av[i] = -expf(al[i]);
      A2[i] = fmaxf(Av[i] * kLog2e, -FLT_MAX);
      iA[i] = -expf(-al[i]);
    }
  }
  // float32: step sizes below this keep the retentions on the near-1
  // polynomial, as in the forward kernels
  const float near_bound = near1_bound(make_float2(A2[0], A2[1]),
                                       make_float2(A2[2], A2[3]));
  (void)near_bound;
  if (ch_ok) {
    if (p.dh_last) {
      const float4 v = *reinterpret_cast<const float4 *>(
          p.dh_last + (b * E + e) * N + 4 * g);
      lam[0] = v.x; lam[1] = v.y; lam[2] = v.z; lam[3] = v.w;
    }
  }
  // the pre-pass channel pair of this thread (THREADS is a multiple of G;
  // E is even, so a pair is wholly inside or wholly past the last channel)
  const int pc = 2 * (tid % (G / 2));
  const int64_t pe = e0 + pc;
  const bool pe_ok = pe < E;
  const float2 pbias = (pe_ok && p.delta_bias)
                           ? make_float2(p.delta_bias[pe], p.delta_bias[pe + 1])
                           : make_float2(0.0f, 0.0f);
  const float Dv = (ch_ok && p.D) ? p.D[e] : 0.0f;
  float sum_dD = 0.0f, sum_db = 0.0f;

  // channel-sum passes: this lane sums history row pr, state quad pq, over
  // the warp's channels j K + pk (j = 0..7), whose slots in the row are the
  // consecutive warp * 32 + 4 j + (lane & 3)
  const int pr = lane >> 2, pq = (lane & 3) % NG, pk = (lane & 3) / NG;
  const float4 *const hrow = sH + (1 + pr) * RS + warp * 32 + (lane & 3);
  const bool warp_ok = e0 + warp * CW < E;
  // add a lane's sum for history row pr of the half at rb into dst [b, L, N]
  // (DET: the block's sum into its slice of the partial array `part`; slot
  // 0 or 1 picks the exchange buffer of the pass)
  float4 *const sRed = reinterpret_cast<float4 *>(smem + Cfg::SMEM_BYTES);
  (void)tile;
  (void)sRed;
  auto red_row = [&](float *dst, float *part, int slot, int64_t t0, int rb,
                     float2 v01, float2 v23) {
    const int64_t t = t0 + rb + pr;
    float4 v = make_float4(v01.x, v01.y, v23.x, v23.y);
    if constexpr (DET) {
      (void)dst;
      // with fewer than 4 state quads, K lanes (bits of lane & 3 above NG)
      // summed different channels of the same row and quad: add theirs
#pragma unroll
      for (int m = NG; m < 4; m <<= 1)
        v = make_float4(v.x + __shfl_xor_sync(FULL, v.x, m),
                        v.y + __shfl_xor_sync(FULL, v.y, m),
                        v.z + __shfl_xor_sync(FULL, v.z, m),
                        v.w + __shfl_xor_sync(FULL, v.w, m));
      // warps 1.. hand their sums to warp 0, which adds them in warp order
      float4 *const sr = sRed + slot * (NW - 1) * 32;
      if (warp > 0) sr[(warp - 1) * 32 + lane] = v;
      __syncthreads();
      if (warp == 0) {
#pragma unroll
        for (int k = 0; k < NW - 1; ++k) {
          const float4 u = sr[k * 32 + lane];
          v = make_float4(v.x + u.x, v.y + u.y, v.z + u.z, v.w + u.w);
        }
        if ((FAST || t < L) && (lane & 3) < NG)
          *reinterpret_cast<float4 *>(
              part + ((tile * p.batch + b) * L + t) * N + 4 * pq) = v;
      }
    } else {
      (void)part;
      (void)slot;
      if (FAST || (warp_ok && t < L))
        atomicAdd(reinterpret_cast<float4 *>(dst + (b * L + t) * N + 4 * pq),
                  v);
    }
  };

  auto stage = [&](int64_t w, int s) {
    unsigned char *base = smem + s * Cfg::STAGE;
    const int64_t t0 = w * TW;
    constexpr int CPR = G * ESZ / 16, EPC = 16 / ESZ;
    for (int idx = tid; idx < TW * CPR; idx += THREADS) {
      const int r = idx / CPR, k = idx - (idx / CPR) * CPR;
      const int64_t t = t0 + r, ec = e0 + k * EPC;
      const bool ok = FAST || (t < L && ec < E);
      const int64_t go = ok ? (b * L + t) * E + ec : 0;
      const int so = r * G * ESZ + k * 16;
      cp_async16(base + so, gx + go, ok);
      cp_async16(base + Cfg::ACT_BYTES + so, gdl + go, ok);
      if (has_z) cp_async16(base + 2 * Cfg::ACT_BYTES + so, gz + go, ok);
      cp_async16(base + 3 * Cfg::ACT_BYTES + so, gdy + go, ok);
    }
    unsigned char *bc = base + 4 * Cfg::ACT_BYTES;
    constexpr int CH = TW * N * ESZ / 16;
    for (int idx = tid; idx < CH; idx += THREADS) {
      const int r = idx * 16 / (N * ESZ);
      const bool ok = FAST || t0 + r < L;
      const int64_t go = ok ? (b * L + t0) * N + int64_t(idx) * (16 / ESZ) : 0;
      cp_async16(bc + idx * 16, gB + go, ok);
      cp_async16(bc + Cfg::BC_BYTES + idx * 16, gC + go, ok);
    }
  };

  // the checkpoints that start window w's two halves, loaded one window
  // ahead so that their latency is hidden behind a window of work
  float4 ck_lo = make_float4(0.0f, 0.0f, 0.0f, 0.0f), ck_hi = ck_lo;
  auto load_ckpts = [&](int64_t w) {
    if (ch_ok) {
      ck_lo = *reinterpret_cast<const float4 *>(
          p.ckpt + ((b * nck + 2 * w) * E + e) * N + 4 * g);
      // the later half may lie wholly past the sequence (no checkpoint, and
      // its steps change nothing): start it from the first one then
      const int64_t k2 = 2 * w + 1 < nck ? 2 * w + 1 : 2 * w;
      ck_hi = *reinterpret_cast<const float4 *>(
          p.ckpt + ((b * nck + k2) * E + e) * N + 4 * g);
    }
  };

  const int64_t w_last = w_hi - 1;
  stage(w_last, 0);
  cp_async_commit();
  load_ckpts(w_last);
  if constexpr (DYN) {
    if (chunk > 0) {
      // the later chunk's hand-over, once published (bounded wait; on
      // timeout the status word says so and this chunk starts from zero)
      const unsigned *flag =
          p.dyn_flags + (b * p.dyn_chunks + chunk - 1) * tiles + tile;
      if (tid == 0) {
        bool ok = false;
        for (unsigned spin = 0; spin < p.spin_limit; ++spin) {
          if (ld_acquire(flag) != 0u) {
            ok = true;
            break;
          }
          __nanosleep(64);
        }
        s_unit = ok ? 1u : 0u;
        if (!ok) atomicExch(p.status, kStatusTimeout);
      }
      __syncthreads();
      const bool got = s_unit != 0u;
      __syncthreads();
      const float *cv =
          p.dyn_carry + ((b * tiles + tile) * THREADS + tid) * 12;
      const float4 u0 = got ? __ldcg(reinterpret_cast<const float4 *>(cv))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 u1 = got ? __ldcg(reinterpret_cast<const float4 *>(cv + 4))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      const float2 u2 = got ? __ldcg(reinterpret_cast<const float2 *>(cv + 8))
                            : make_float2(0.f, 0.f);
      lam[0] = u0.x; lam[1] = u0.y; lam[2] = u0.z; lam[3] = u0.w;
      dA[0] = u1.x; dA[1] = u1.y; dA[2] = u1.z; dA[3] = u1.w;
      sum_dD = u2.x;
      sum_db = u2.y;
    }
  }
  for (int64_t w = w_last; w >= w_lo; --w) {
    const int par = int((w_last - w) & 1);
    // this window's tiles have landed, and every thread is done with the
    // previous window, whose buffer now takes the next window's tiles
    cp_async_wait<0>();
    __syncthreads();
    if (w > w_lo) stage(w - 1, par ^ 1);
    cp_async_commit();

    const int64_t t0 = w * TW;
    const unsigned char *base = smem + par * Cfg::STAGE;
    const T *const sBr = reinterpret_cast<const T *>(base + 4 * Cfg::ACT_BYTES);
    const T *const sCr = reinterpret_cast<const T *>(
        base + 4 * Cfg::ACT_BYTES + Cfg::BC_BYTES);
    // ---- 2. per (t, e) scalars, once, for two adjacent channels at a time.
    // The staged tiles are zero past the sequence and past the last channel,
    // which makes x, dy and the gate slope zero there; the step size is set
    // to zero past the sequence, so that those steps leave lam unchanged.
    for (int idx = tid; idx < TW * (G / 2); idx += THREADS) {
      int r = idx / (G / 2);  // 2 (idx % (G / 2)) == pc
      if constexpr (G == 16) {
        // a warp covers 4 rows, 8 lanes each: let each half-warp store rows
        // r and r + 2, whose 8-byte stores fall 16 banks apart (rows r and
        // r + 1 would share 8 of their banks at this row stride)
        const int q = r & 3;
        r = (r & ~3) | ((q & 1) << 1) | (q >> 1);
      }
      const int o = (r * G + pc) * ESZ;
      const float2 raw = add2(
          Act<T>::load2(reinterpret_cast<const T *>(base + Cfg::ACT_BYTES + o)),
          pbias);
      const float2 xv = Act<T>::load2(reinterpret_cast<const T *>(base + o));
      const float2 gv = Act<T>::load2(
          reinterpret_cast<const T *>(base + 3 * Cfg::ACT_BYTES + o));
      float2 dyv = gv, gzv = make_float2(0.0f, 0.0f);
      if (has_z) {
        // y = pre SiLU(z): dy = g SiLU(z), dz = g pre sg (1 + z (1 - sg))
        const float2 zv = Act<T>::load2(
            reinterpret_cast<const T *>(base + 2 * Cfg::ACT_BYTES + o));
        const float2 sg = PairMath<T>::sigmoid(zv);
        const float2 gs = mul2(gv, sg);
        dyv = mul2(gs, zv);
        gzv = mul2(gs, fma2(zv, add2(make_float2(1.0f, 1.0f),
                                     make_float2(-sg.x, -sg.y)),
                            make_float2(1.0f, 1.0f)));
      }
      float2 sv = raw, slope = make_float2(1.0f, 1.0f);
      if (FAST || p.softplus) PairMath<T>::softplus_slope(raw, sv, slope);
      const bool ok = FAST || t0 + r < L;
      const int so = r * SP + pc;
      *reinterpret_cast<float2 *>(sS + so) = ok ? sv : make_float2(0.0f, 0.0f);
      *reinterpret_cast<float2 *>(sX + so) = xv;
      *reinterpret_cast<float2 *>(sDY + so) = dyv;
      *reinterpret_cast<float2 *>(sGZ + so) = gzv;
      *reinterpret_cast<float2 *>(sSG + so) = slope;
    }
    __syncthreads();

    // ---- 3. recompute this lane's states from the checkpoints, half a
    // window (one checkpoint interval) at a time, the later half first: the
    // state history of the half being reversed is kept in shared memory.
    // Both halves start from a stored state, so each step is recomputed once.
    // (this window's checkpoints were loaded during the previous window)
    const float hck[4] = {ck_lo.x, ck_lo.y, ck_lo.z, ck_lo.w};
    const float hmid[4] = {ck_hi.x, ck_hi.y, ck_hi.z, ck_hi.w};
    if (w > w_lo) load_ckpts(w - 1);
    // advance h over rows [r0, r0 + HALF); STORE: keep each state in sH
    // (row 1 + r - r0)
    auto recompute = [&](float (&h)[4], int r0, bool store) {
#pragma unroll
      for (int r = r0; r < r0 + HALF; ++r) {
        const float sv = sS[r * SP + cl];
        const float xv = sX[r * SP + cl];
        const float4 Bq = Act<T>::load4(sBr + r * N + 4 * g);
        if constexpr (ZOH) {
          const float Bv[4] = {Bq.x, Bq.y, Bq.z, Bq.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float zl = sv * A2[i];
            const float a = sizeof(T) == 4 ? retention_f32(zl) : ex2(zl);
            h[i] = fmaf(a, h[i], zoh_factor(sv, zl, a, iA[i]) * xv * Bv[i]);
          }
        } else {  // packed pairs: a = 2^(s A'), h = a h + (s x) B
          const float2 s2 = make_float2(sv, sv);
          const float2 sx2 = make_float2(sv * xv, sv * xv);
          const float2 zl01 = mul2(s2, make_float2(A2[0], A2[1]));
          const float2 zl23 = mul2(s2, make_float2(A2[2], A2[3]));
          float2 a01 = ex2x2(zl01), a23 = ex2x2(zl23);
          if constexpr (sizeof(T) == 4)
            near1_retentions(sv, near_bound, zl01, zl23, a01, a23);
          const float2 h01 = fma2(a01, make_float2(h[0], h[1]),
                                  mul2(sx2, make_float2(Bq.x, Bq.y)));
          const float2 h23 = fma2(a23, make_float2(h[2], h[3]),
                                  mul2(sx2, make_float2(Bq.z, Bq.w)));
          h[0] = h01.x; h[1] = h01.y; h[2] = h23.x; h[3] = h23.y;
        }
        if (store)
          sH[(1 + r - r0) * RS + tid] = make_float4(h[0], h[1], h[2], h[3]);
      }
    };
#pragma unroll 1
    for (int half = 1; half >= 0; --half) {
      const int rb = half * HALF;
      float hst[4];  // the state before row rb
#pragma unroll
      for (int i = 0; i < 4; ++i) hst[i] = half ? hmid[i] : hck[i];
      sH[tid] = make_float4(hst[0], hst[1], hst[2], hst[3]);
      // the state after step r of the sweep below, carried from the previous
      // (later) step; the recompute leaves the half's last state
      float4 hc;
      {
        float h[4] = {hst[0], hst[1], hst[2], hst[3]};
        recompute(h, rb, true);
        hc = make_float4(h[0], h[1], h[2], h[3]);
      }
      __syncwarp();
      // dC[t, n] = sum_e dy h_t[e, n], over this warp's channels
      {
        const float *dyr = sDY + (rb + pr) * SP + warp * CW + pk;
        float dyv[8];
        if constexpr (K == 1) {
          const float4 d0 = *reinterpret_cast<const float4 *>(dyr);
          const float4 d1 = *reinterpret_cast<const float4 *>(dyr + 4);
          dyv[0] = d0.x; dyv[1] = d0.y; dyv[2] = d0.z; dyv[3] = d0.w;
          dyv[4] = d1.x; dyv[5] = d1.y; dyv[6] = d1.z; dyv[7] = d1.w;
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) dyv[j] = dyr[j * K];
        }
        float2 c01 = make_float2(0.0f, 0.0f), c23 = c01;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 hv = hrow[4 * j];
          const float2 d2 = make_float2(dyv[j], dyv[j]);
          c01 = fma2(d2, make_float2(hv.x, hv.y), c01);
          c23 = fma2(d2, make_float2(hv.z, hv.w), c23);
        }
        red_row(p.dC, p.part_dC, 0, t0, rb, c01, c23);
      }
      __syncwarp();

      // ---- 4. the reverse sweep over the half, in blocks of NG steps: the
      // per-channel sums (C.h, the dx and d-step partials) are off the
      // adjoint's critical path, so they are kept per step and summed over
      // the channel's lanes once per block by a transposing butterfly that
      // leaves lane g the totals of the block's step g, which it finishes
#pragma unroll
      for (int jb = HALF / NG - 1; jb >= 0; --jb) {
        float pre_s[NG], dxp_s[NG], dsp_s[NG];
#pragma unroll
        for (int s = NG - 1; s >= 0; --s) {
          const int r = rb + jb * NG + s;
          const float4 hp4 = sH[(r - rb) * RS + tid];
          const float hcur[4] = {hc.x, hc.y, hc.z, hc.w};
          const float hprev[4] = {hp4.x, hp4.y, hp4.z, hp4.w};
          const float sv = sS[r * SP + cl];
          const float xv = sX[r * SP + cl];
          const float dyv = sDY[r * SP + cl];
          const float4 Bq = Act<T>::load4(sBr + r * N + 4 * g);
          const float4 Cq = Act<T>::load4(sCr + r * N + 4 * g);
          const float Bv[4] = {Bq.x, Bq.y, Bq.z, Bq.w};
          const float Cv[4] = {Cq.x, Cq.y, Cq.z, Cq.w};
          float &pre = pre_s[s], &dxp = dxp_s[s], &dsp = dsp_s[s];
          pre = dxp = dsp = 0.0f;
          float4 dBq;  // this step's lam f x, summed into dB after the sweep
          if constexpr (!ZOH) {
            // packed pairs of states; sum_n lam B gives both the dx and the
            // write part of the step-size partial: dx = s sum lam B,
            // d step = x sum lam B + sum (lam h_{t-1} a) A
            const float2 s2 = make_float2(sv, sv), dy2 = make_float2(dyv, dyv);
            const float2 hc01 = make_float2(hcur[0], hcur[1]);
            const float2 hc23 = make_float2(hcur[2], hcur[3]);
            const float2 B01 = make_float2(Bv[0], Bv[1]);
            const float2 B23 = make_float2(Bv[2], Bv[3]);
            const float2 C01 = make_float2(Cv[0], Cv[1]);
            const float2 C23 = make_float2(Cv[2], Cv[3]);
            const float2 zl01 = mul2(s2, make_float2(A2[0], A2[1]));
            const float2 zl23 = mul2(s2, make_float2(A2[2], A2[3]));
            float2 a01 = ex2x2(zl01), a23 = ex2x2(zl23);
            if constexpr (sizeof(T) == 4)
              near1_retentions(sv, near_bound, zl01, zl23, a01, a23);
            const float2 ch = fma2(C23, hc23, mul2(C01, hc01));
            pre = ch.x + ch.y;
            float2 l01 = fma2(dy2, C01, make_float2(lam[0], lam[1]));
            float2 l23 = fma2(dy2, C23, make_float2(lam[2], lam[3]));
            const float2 lb = fma2(l23, B23, mul2(l01, B01));
            const float slb = lb.x + lb.y;
            const float2 sx2 = make_float2(sv * xv, sv * xv);
            const float2 dB01 = mul2(l01, sx2), dB23 = mul2(l23, sx2);
            const float2 g01 =
                mul2(mul2(l01, make_float2(hprev[0], hprev[1])), a01);
            const float2 g23 =
                mul2(mul2(l23, make_float2(hprev[2], hprev[3])), a23);
            const float2 gA = fma2(g23, make_float2(Av[2], Av[3]),
                                   mul2(g01, make_float2(Av[0], Av[1])));
            dsp = fmaf(xv, slb, gA.x + gA.y);
            dxp = sv * slb;
            const float2 dA01 = fma2(g01, s2, make_float2(dA[0], dA[1]));
            const float2 dA23 = fma2(g23, s2, make_float2(dA[2], dA[3]));
            dA[0] = dA01.x; dA[1] = dA01.y; dA[2] = dA23.x; dA[3] = dA23.y;
            l01 = mul2(l01, a01);
            l23 = mul2(l23, a23);
            lam[0] = l01.x; lam[1] = l01.y; lam[2] = l23.x; lam[3] = l23.y;
            dBq = make_float4(dB01.x, dB01.y, dB23.x, dB23.y);
          } else {  // zero-order-hold write f = expm1(s A) / A, per state
            float dBv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float zl = sv * A2[i];
              const float a = sizeof(T) == 4 ? retention_f32(zl) : ex2(zl);
              pre = fmaf(Cv[i], hcur[i], pre);
              lam[i] = fmaf(dyv, Cv[i], lam[i]);
              const float da = lam[i] * hprev[i];
              const float f = zoh_factor(sv, zl, a, iA[i]);
              const float lbx = lam[i] * Bv[i] * xv;
              dsp = fmaf(lbx, a, dsp);
              dBv[i] = lam[i] * f * xv;
              dxp = fmaf(lam[i] * f, Bv[i], dxp);
              dA[i] = fmaf(lbx, (sv * a - f) * iA[i], dA[i]);
              dsp = fmaf(da * a, Av[i], dsp);
              dA[i] = fmaf(da * a, sv, dA[i]);
              lam[i] *= a;
            }
            dBq = make_float4(dBv[0], dBv[1], dBv[2], dBv[3]);
          }
          // step r's history slot is not read again: it takes the dB terms
          sH[(1 + r - rb) * RS + tid] = dBq;
          hc = hp4;
        }
        const float pre = transpose_reduce<NG, 1>(pre_s, g);
        const float dxp = transpose_reduce<NG, 1>(dxp_s, g);
        const float dsp = transpose_reduce<NG, 1>(dsp_s, g);
        const int r = rb + jb * NG + g;
        const int64_t t = t0 + r;
        if (FAST || (ch_ok && t < L)) {
          const int64_t i = (b * L + t) * E + e;
          const float dyv = sDY[r * SP + cl];
          const float xv = sX[r * SP + cl];
          const float dxv = fmaf(dyv, Dv, dxp);
          const float draw = dsp * sSG[r * SP + cl];
          Act<T>::store(static_cast<T *>(p.dx) + i, dxv);
          Act<T>::store(static_cast<T *>(p.ddelta) + i, draw);
          if (has_z)
            Act<T>::store(static_cast<T *>(p.dz) + i,
                          sGZ[r * SP + cl] * fmaf(Dv, xv, pre));
          sum_dD = fmaf(dyv, xv, sum_dD);
          sum_db += draw;
        }
      }
      __syncwarp();
      // dB[t, n] = sum_e lam f x, over this warp's channels
      {
        float2 b01 = make_float2(0.0f, 0.0f), b23 = b01;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 v = hrow[4 * j];
          b01 = add2(b01, make_float2(v.x, v.y));
          b23 = add2(b23, make_float2(v.z, v.w));
        }
        red_row(p.dB, p.part_dB, 1, t0, rb, b01, b23);
      }
      __syncwarp();
    }
  }
  cp_async_wait<0>();
  if constexpr (DYN) {
    if (w_lo > 0) {  // an earlier chunk goes on from here
      float *const cv =
          p.dyn_carry + ((b * tiles + tile) * THREADS + tid) * 12;
      __stcg(reinterpret_cast<float4 *>(cv),
             make_float4(lam[0], lam[1], lam[2], lam[3]));
      __stcg(reinterpret_cast<float4 *>(cv + 4),
             make_float4(dA[0], dA[1], dA[2], dA[3]));
      __stcg(reinterpret_cast<float2 *>(cv + 8), make_float2(sum_dD, sum_db));
      __threadfence();
      __syncthreads();
      if (tid == 0 && !((p.debug & kDebugNoPublish) && chunk == 0))
        st_release(p.dyn_flags + (b * p.dyn_chunks + chunk) * tiles + tile,
                   1u);
      continue;
    }
  }
  // every lane of a channel finished some of its steps: sum the partials
#pragma unroll
  for (int m = 1; m < NG; m <<= 1) {
    sum_dD += __shfl_xor_sync(FULL, sum_dD, m);
    sum_db += __shfl_xor_sync(FULL, sum_db, m);
  }

  if (ch_ok) {
    if (p.dh0)
      *reinterpret_cast<float4 *>(p.dh0 + (b * E + e) * N + 4 * g) =
          make_float4(lam[0], lam[1], lam[2], lam[3]);
    if constexpr (DET) {  // this batch row's share, summed afterwards
      *reinterpret_cast<float4 *>(p.part_dA + (b * E + e) * N + 4 * g) =
          make_float4(dA[0] * Av[0], dA[1] * Av[1], dA[2] * Av[2],
                      dA[3] * Av[3]);
      if (g == 0) {
        if (p.dD) p.part_dD[b * E + e] = sum_dD;
        if (p.ddelta_bias) p.part_db[b * E + e] = sum_db;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        atomicAdd(p.dA_log + e * N + 4 * g + i, dA[i] * Av[i]);
      if (g == 0) {
        if (p.dD) atomicAdd(p.dD + e, sum_dD);
        if (p.ddelta_bias) atomicAdd(p.ddelta_bias + e, sum_db);
      }
    }
  }
  if constexpr (!DYN) break;
  }  // the DYN pass loop
}

// out[i] = sum over k = 0 .. slices-1, in that order, of part[k n + i]; n a
// multiple of 4. The deterministic backward's last step.
constexpr int kBwdRedBytes = 2 * 32 * 16;  // DET exchange, per extra warp
__global__ void __launch_bounds__(256)
    sum_slices_kernel(const float *part, int64_t slices, int64_t n,
                      float *out) {
  const int64_t n4 = n / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int64_t k = 0; k < slices; ++k) {
      const float4 v = __ldcs(reinterpret_cast<const float4 *>(part + k * n) + i);
      acc = make_float4(acc.x + v.x, acc.y + v.y, acc.z + v.z, acc.w + v.w);
    }
    reinterpret_cast<float4 *>(out)[i] = acc;
  }
}

}  // namespace ssm
