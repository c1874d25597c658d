// Device-side arithmetic shared by the scan kernels: hardware exp2/log2/rcp
// through the SFU (MUFU) pipe, the step-size softplus, the SiLU gate and
// activation loads/stores for float32 and bfloat16.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace ssm {

constexpr float kLog2e = 1.4426950408889634f;  // 1 / ln 2
constexpr float kLn2 = 0.6931471805599453f;

// 2^x on the SFU (one MUFU.EX2). Flushes subnormal results to zero, so a
// retention exp(delta*A) below 2^-126 becomes exactly 0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log2(x) on the SFU (one MUFU.LG2).
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 1/x on the SFU (one MUFU.RCP); 1/inf = 0.
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log(1 + u) for u in [0, 1]. Below 1/8 the alternating Taylor series
// u - u^2/2 + u^3/3 - ... truncated after the u^8 term (relative truncation
// error < u^8 / 9 < 2^-27), evaluated in Estrin's grouping (dependency depth
// 4 instead of 8):
//   u [ (1 - u/2) + u^2 (1/3 - u/4) + u^4 ((1/5 - u/6) + u^2 (1/7 - u/8)) ].
// From 1/8 up, log2(1 + u) * ln 2, where rounding 1 + u costs at most 2^-24
// absolute, i.e. < 5e-7 relative to log(1.125).
__device__ __forceinline__ float log1p_unit(float u) {
  const float u2 = u * u;
  const float u4 = u2 * u2;
  const float p0 = fmaf(u, -0.5f, 1.0f);
  const float p1 = fmaf(u, -0.25f, 0.3333333333333333f);
  const float p2 = fmaf(u, -0.16666666666666666f, 0.2f);
  const float p3 = fmaf(u, -0.125f, 0.14285714285714285f);
  const float q0 = fmaf(u2, p1, p0);
  const float q1 = fmaf(u2, p3, p2);
  const float s = fmaf(u4, q1, q0) * u;
  const float l = lg2(1.0f + u) * kLn2;
  return u < 0.125f ? s : l;
}

// softplus with PyTorch's default threshold: v for v > 20, else
// log(1 + e^v) = max(v, 0) + log(1 + e^-|v|), which never overflows and keeps
// relative accuracy for very negative v (where the result is ~e^v).
__device__ __forceinline__ float softplus(float v) {
  const float u = ex2(-fabsf(v) * kLog2e);  // e^-|v| in (0, 1]
  const float r = fmaxf(v, 0.0f) + log1p_unit(u);
  return v > 20.0f ? v : r;
}

// SiLU(z) = z * sigmoid(z) = z / (1 + e^-z). For z -> -inf, e^-z = inf and
// rcp(inf) = 0 gives -0; for z -> +inf it gives z.
__device__ __forceinline__ float silu(float z) {
  return z * rcp(1.0f + ex2(-z * kLog2e));
}

// Packed float32 pairs (Blackwell FFMA2 / FMUL2): one instruction issues two
// independent float32 operations, each rounded as its scalar form would be.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rc, rd;\n"
      " mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n"
      " mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n"
      " mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 ex2x2(float2 v) {
  return make_float2(ex2(v.x), ex2(v.y));
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n"
      " mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// softplus of two values at once: the same formula as softplus(), with the
// series and the bookkeeping on packed pairs.
__device__ __forceinline__ float2 softplus2(float2 v) {
  const float2 u = make_float2(ex2(-fabsf(v.x) * kLog2e),
                               ex2(-fabsf(v.y) * kLog2e));
  const float2 u2 = mul2(u, u);
  const float2 u4 = mul2(u2, u2);
  const float2 p0 = fma2(u, make_float2(-0.5f, -0.5f), make_float2(1.0f, 1.0f));
  const float2 p1 = fma2(u, make_float2(-0.25f, -0.25f),
                         make_float2(0.3333333333333333f, 0.3333333333333333f));
  const float2 p2 = fma2(u, make_float2(-0.16666666666666666f,
                                        -0.16666666666666666f),
                         make_float2(0.2f, 0.2f));
  const float2 p3 = fma2(u, make_float2(-0.125f, -0.125f),
                         make_float2(0.14285714285714285f, 0.14285714285714285f));
  const float2 s = mul2(fma2(u4, fma2(u2, p3, p2), fma2(u2, p1, p0)), u);
  const float2 w = add2(u, make_float2(1.0f, 1.0f));
  const float2 l = mul2(make_float2(lg2(w.x), lg2(w.y)), make_float2(kLn2, kLn2));
  const float2 lp = make_float2(u.x < 0.125f ? s.x : l.x,
                                u.y < 0.125f ? s.y : l.y);
  const float2 r = add2(make_float2(fmaxf(v.x, 0.0f), fmaxf(v.y, 0.0f)), lp);
  return make_float2(v.x > 20.0f ? v.x : r.x, v.y > 20.0f ? v.y : r.y);
}

// SiLU of two values at once.
__device__ __forceinline__ float2 silu2(float2 z) {
  const float2 e = mul2(z, make_float2(-kLog2e, -kLog2e));
  const float2 d = add2(make_float2(ex2(e.x), ex2(e.y)), make_float2(1.0f, 1.0f));
  return mul2(z, make_float2(rcp(d.x), rcp(d.y)));
}

// tanh on the SFU (one MUFU.TANH; relative error about 2^-11).
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Cheaper forms for bfloat16 activations, whose inputs already carry a
// relative rounding of 2^-9:
// softplus as log2(1 + 2^(v log2 e)) ln 2 (2 MUFU, no series). Rounding
// 1 + e^v and the SFU log cost at most ~3e-7 absolute, which is what is left
// of a very negative v's e^v; PyTorch's threshold (v above 20) is kept.
__device__ __forceinline__ float2 softplus2_fast(float2 v) {
  const float2 e = mul2(v, make_float2(kLog2e, kLog2e));
  const float2 w = add2(make_float2(ex2(e.x), ex2(e.y)),
                        make_float2(1.0f, 1.0f));
  const float2 r =
      mul2(make_float2(lg2(w.x), lg2(w.y)), make_float2(kLn2, kLn2));
  return make_float2(v.x > 20.0f ? v.x : r.x, v.y > 20.0f ? v.y : r.y);
}

// SiLU as h + h tanh(h), h = z/2 (z sigmoid(z) with sigmoid(z) =
// (1 + tanh(z/2)) / 2): 1 MUFU, absolute error of the sigmoid below 2.5e-4.
__device__ __forceinline__ float2 silu2_fast(float2 z) {
  const float2 h = mul2(z, make_float2(0.5f, 0.5f));
  return fma2(h, make_float2(tanh_approx(h.x), tanh_approx(h.y)), h);
}

// sigmoid(v) = 1 / (1 + e^-v) of two values; 0 for v -> -inf, 1 for +inf.
__device__ __forceinline__ float2 sigmoid2(float2 v) {
  const float2 e = mul2(v, make_float2(-kLog2e, -kLog2e));
  const float2 d = add2(make_float2(ex2(e.x), ex2(e.y)), make_float2(1.0f, 1.0f));
  return make_float2(rcp(d.x), rcp(d.y));
}

// The step-size softplus and the SiLU the chunked kernel applies to packed
// pairs: exact-rounding-order forms for float32 activations, the cheaper
// forms above for bfloat16. The backward pass takes their derivatives from
// the same forms: softplus_slope gives softplus(v) and sigmoid(v) (its
// slope); sigmoid(z) is the gate's, SiLU(z) = z sigmoid(z).
template <typename T> struct PairMath {
  static __device__ __forceinline__ float2 softplus(float2 v) {
    return softplus2(v);
  }
  static __device__ __forceinline__ float2 silu(float2 z) { return silu2(z); }
  static __device__ __forceinline__ void softplus_slope(float2 v, float2 &sp,
                                                        float2 &slope) {
    sp = softplus2(v);
    slope = sigmoid2(v);
  }
  static __device__ __forceinline__ float2 sigmoid(float2 z) {
    return sigmoid2(z);
  }
};
template <> struct PairMath<__nv_bfloat16> {
  static __device__ __forceinline__ float2 softplus(float2 v) {
    return softplus2_fast(v);
  }
  static __device__ __forceinline__ float2 silu(float2 z) {
    return silu2_fast(z);
  }
  // softplus2_fast's value, and its slope e^v / (1 + e^v) from the same e^v
  // (a product, so it keeps relative accuracy where e^v is tiny); above the
  // threshold the value is v and the slope 1.
  static __device__ __forceinline__ void softplus_slope(float2 v, float2 &sp,
                                                        float2 &slope) {
    const float2 e2 = mul2(v, make_float2(kLog2e, kLog2e));
    const float2 e = make_float2(ex2(e2.x), ex2(e2.y));
    const float2 w = add2(e, make_float2(1.0f, 1.0f));
    const float2 r =
        mul2(make_float2(lg2(w.x), lg2(w.y)), make_float2(kLn2, kLn2));
    const float2 sl = mul2(e, make_float2(rcp(w.x), rcp(w.y)));
    sp = make_float2(v.x > 20.0f ? v.x : r.x, v.y > 20.0f ? v.y : r.y);
    slope = make_float2(v.x > 20.0f ? 1.0f : sl.x, v.y > 20.0f ? 1.0f : sl.y);
  }
  // (1 + tanh(z/2)) / 2, the sigmoid inside silu2_fast
  static __device__ __forceinline__ float2 sigmoid(float2 z) {
    const float2 h = mul2(z, make_float2(0.5f, 0.5f));
    return fma2(make_float2(tanh_approx(h.x), tanh_approx(h.y)),
                make_float2(0.5f, 0.5f), make_float2(0.5f, 0.5f));
  }
};

// Retentions close to 1 for float32 activations. The SFU's exp2 errs by up to
// about 1.4 units in the last place near 1, and a retention that repeats
// step after step (a held input) compounds that error linearly over the
// state's memory, about 1/|z| steps. Where |z| = |delta A| < 2^-8 the
// retention is instead the Taylor polynomial 1 + z + z^2/2 (truncation below
// |z|^3/6 < 1e-8, a sixth of a unit in the last place), rounded once by its
// final fused multiply-add. It is written in zl = z log2(e):
// e^z = 1 + zl (c1 + zl c2), c1 = ln 2, c2 = (ln 2)^2 / 2.
constexpr float kNear1Zl = 0.0056355275034725f;  // 2^-8 / ln 2
constexpr float kNear1C1 = 0.6931471805599453f;
constexpr float kNear1C2 = 0.2402265069591007f;

// The per-lane step-size bound below which all four of a lane's states are
// in the polynomial's band: kNear1Zl / max_n |A'_n| (A' = A log2 e, <= 0).
__device__ __forceinline__ float near1_bound(float2 A01, float2 A23) {
  const float m = fmaxf(fmaxf(-A01.x, -A01.y), fmaxf(-A23.x, -A23.y));
  return kNear1Zl / m;  // +inf when every A is 0
}

// For one step of four states (two packed pairs): when |d| < bound, replace
// the SFU retentions a01, a23 (of arguments zl01, zl23) by the polynomial.
// One comparison per step and lane; the polynomial runs on packed pairs and
// only its last multiply-add is predicated.
__device__ __forceinline__ void near1_retentions(float d, float bound,
                                                 float2 zl01, float2 zl23,
                                                 float2 &a01, float2 &a23) {
  asm("{\n"
      " .reg .pred p;\n"
      " .reg .f32 ad;\n"
      " .reg .b64 z0, z1, t0, t1, r0, r1, c1, c2, one;\n"
      " abs.f32 ad, %4;\n"
      " setp.lt.f32 p, ad, %5;\n"
      " mov.b64 z0, {%6, %7};\n"
      " mov.b64 z1, {%8, %9};\n"
      " mov.b64 c2, {%10, %10};\n"
      " mov.b64 c1, {%11, %11};\n"
      " mov.b64 one, {%12, %12};\n"
      " mov.b64 r0, {%0, %1};\n"
      " mov.b64 r1, {%2, %3};\n"
      " fma.rn.f32x2 t0, z0, c2, c1;\n"
      " fma.rn.f32x2 t1, z1, c2, c1;\n"
      " @p fma.rn.f32x2 r0, z0, t0, one;\n"
      " @p fma.rn.f32x2 r1, z1, t1, one;\n"
      " mov.b64 {%0, %1}, r0;\n"
      " mov.b64 {%2, %3}, r1;\n"
      "}"
      : "+f"(a01.x), "+f"(a01.y), "+f"(a23.x), "+f"(a23.y)
      : "f"(d), "f"(bound), "f"(zl01.x), "f"(zl01.y), "f"(zl23.x),
        "f"(zl23.y), "f"(kNear1C2), "f"(kNear1C1), "f"(1.0f));
}

// near1_retentions for a step that the whole warp takes together: the
// polynomial is skipped, by a branch every lane takes the same way, when no
// lane of the warp has a step size in the band. Call it with all 32 lanes.
__device__ __forceinline__ void near1_retentions_warp(float d, float bound,
                                                      float2 zl01, float2 zl23,
                                                      float2 &a01,
                                                      float2 &a23) {
  if (__any_sync(0xffffffffu, fabsf(d) < bound))
    near1_retentions(d, bound, zl01, zl23, a01, a23);
}

// The same for one state (scalar kernels): e^z for zl = z log2 e.
__device__ __forceinline__ float retention_f32(float zl) {
  const float a = ex2(zl);
  const float p = fmaf(zl, fmaf(zl, kNear1C2, kNear1C1), 1.0f);
  return fabsf(zl) < kNear1Zl ? p : a;
}

// Exact zero-order-hold write factor expm1(z) / A, z = d A, for one state:
// given zl = z log2(e) (so a = 2^zl) and invA = 1/A. For |z| < 1/8 it is
// d phi(z) with phi(z) = (e^z - 1)/z = 1 + z/2 + z^2/6 + z^3/24 + z^4/120 +
// z^5/720 (truncation below z^6/5040 < 8e-10 relative); otherwise (a - 1)/A,
// where |a - 1| >= 1 - e^(-1/8) = 0.1175 keeps the subtraction accurate.
__device__ __forceinline__ float zoh_factor(float d, float zl, float a,
                                            float invA) {
  const float z = zl * kLn2;
  float ph = fmaf(z, 1.0f / 720.0f, 1.0f / 120.0f);
  ph = fmaf(z, ph, 1.0f / 24.0f);
  ph = fmaf(z, ph, 1.0f / 6.0f);
  ph = fmaf(z, ph, 0.5f);
  ph = fmaf(z, ph, 1.0f);
  return fabsf(z) < 0.125f ? d * ph : (a - 1.0f) * invA;
}

// The same for two states at once (packed pairs).
__device__ __forceinline__ float2 zoh_factor2(float2 d, float2 zl, float2 a,
                                              float2 invA) {
  const float2 z = mul2(zl, make_float2(kLn2, kLn2));
  float2 ph = fma2(z, make_float2(1.0f / 720.0f, 1.0f / 720.0f),
                   make_float2(1.0f / 120.0f, 1.0f / 120.0f));
  ph = fma2(z, ph, make_float2(1.0f / 24.0f, 1.0f / 24.0f));
  ph = fma2(z, ph, make_float2(1.0f / 6.0f, 1.0f / 6.0f));
  ph = fma2(z, ph, make_float2(0.5f, 0.5f));
  ph = fma2(z, ph, make_float2(1.0f, 1.0f));
  const float2 sm = mul2(d, ph);
  const float2 lg = mul2(add2(a, make_float2(-1.0f, -1.0f)), invA);
  return make_float2(fabsf(z.x) < 0.125f ? sm.x : lg.x,
                     fabsf(z.y) < 0.125f ? sm.y : lg.y);
}

template <typename T> struct Act;

template <> struct Act<float> {
  static __device__ __forceinline__ float load(const float *p) { return *p; }
  // two adjacent elements (8-byte aligned)
  static __device__ __forceinline__ float2 load2(const float *p) {
    return *reinterpret_cast<const float2 *>(p);
  }
  // four adjacent elements (16-byte aligned)
  static __device__ __forceinline__ float4 load4(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
  }
  static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
};

template <> struct Act<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
    return __bfloat162float(*p);
  }
  // two adjacent elements (4-byte aligned)
  static __device__ __forceinline__ float2 load2(const __nv_bfloat16 *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
  }
  // four adjacent elements (8-byte aligned) in one 8-byte load; a bfloat16
  // is the upper half of the float32 with the same value
  static __device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(u.x << 16),
                       __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) {
    *p = __float2bfloat16_rn(v);
  }
};

}  // namespace ssm
