// Shared device helpers of the FNO CUDA library (sm_100a).
//
// Conventions follow the block definition in include/fno.h: forward transform
// exp(-i theta), inverse exp(+i theta), kept modes per axis "positive block
// then negative block" on non-last axes and 0..m-1 on the last axis.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fno {

// ---------------------------------------------------------------------------
// storage dtype <-> float
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T> __device__ __forceinline__ float ldf(const T *p) { return to_f<T>(p[0]); }
template <> __device__ __forceinline__ float ldf<float>(const float *p) { return __ldg(p); }

// complex value stored as two consecutive storage elements (re, im)
template <typename T> __device__ __forceinline__ float2 ldc(const T *p) {
  return make_float2(to_f<T>(p[0]), to_f<T>(p[1]));
}
template <> __device__ __forceinline__ float2 ldc<float>(const float *p) {
  return __ldg(reinterpret_cast<const float2 *>(p));
}

// ---------------------------------------------------------------------------
// complex arithmetic on float2 (x = re, y = im)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
// a += b * c
__device__ __forceinline__ void cfma(float2 &a, float2 b, float2 c) {
  a.x = fmaf(b.x, c.x, fmaf(-b.y, c.y, a.x));
  a.y = fmaf(b.x, c.y, fmaf(b.y, c.x, a.y));
}
// a += conj(b) * c
__device__ __forceinline__ void cfma_conj_a(float2 &a, float2 b, float2 c) {
  a.x = fmaf(b.x, c.x, fmaf(b.y, c.y, a.x));
  a.y = fmaf(b.x, c.y, fmaf(-b.y, c.x, a.y));
}
// a += b * conj(c)
__device__ __forceinline__ void cfma_conj_b(float2 &a, float2 b, float2 c) {
  a.x = fmaf(b.x, c.x, fmaf(b.y, c.y, a.x));
  a.y = fmaf(b.y, c.x, fmaf(-b.x, c.y, a.y));
}

// ---------------------------------------------------------------------------
// twiddles: tw[j] = (cos, sin)(2 pi j / N), j in [0, N), built in double
// precision and rounded once, so every table entry is correctly rounded.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void build_twiddles(float2 *tw, int n) {
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    int jj = (2 * j > n) ? j - n : j;  // angle in (-pi, pi]
    double s, c;
    sincospi(2.0 * (double)jj / (double)n, &s, &c);
    tw[j] = make_float2((float)c, (float)s);
  }
}

// kept wavenumber of storage slot q on a non-last axis (positive block first)
__device__ __forceinline__ int kept_k(int q, int m, int n) { return q < m ? q : n - 2 * m + q; }

// (k * r) mod n for 0 <= k, r < n <= 4096 (fits in 32 bits)
__device__ __forceinline__ int mulmod(int k, int r, int n) { return (k * r) % n; }

// Walks the twiddle index (kept_k(q, m, n) * r) mod n over q = 0, 1, ...:
// the positive block starts at 0 and the negative block at ((n - m) r) mod n,
// each advancing by r.  With m == 0 (a single kept mode, k = 0) it stays 0.
struct KeptIndex {
  int idx, step, n, m, q;
  __device__ __forceinline__ KeptIndex(int m_, int n_, int r) : idx(0), step(r % n_), n(n_), m(m_), q(0) {}
  __device__ __forceinline__ int next() {
    const int cur = idx;
    ++q;
    if (q == m) {
      idx = mulmod(n - m, step, n);
    } else {
      idx += step;
      if (idx >= n) idx -= n;
    }
    return cur;
  }
};

// ---------------------------------------------------------------------------
// activations
// ---------------------------------------------------------------------------
// erf by Hastings' approximation (Abramowitz and Stegun, Handbook of
// Mathematical Functions, formula 7.1.28): for t >= 0
//   erf t = 1 - (1 + a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5 + a6 t^6)^-16
// with |error| <= 3e-7.  Horner's rule, four squarings and one approximate
// reciprocal; a power that overflows gives erfc = 0.  No branches, so the
// GELUs of a thread's channels interleave freely.
constexpr float kErfA1 = 0.0705230784f, kErfA2 = 0.0422820123f, kErfA3 = 0.0092705272f,
                kErfA4 = 0.0001520143f, kErfA5 = 0.0002765672f, kErfA6 = 0.0000430638f;

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// erfc(t) = 1 - erf(t) for t >= 0.  The power is carried as v = q - 1
// (each squaring v <- v (v + 2)), so near t = 0, where q is close to 1, the
// rounding of q is not raised to the 16th power: Phi = erfc / 2 is within
// 2.5e-7 in float32 (the formula's own 1.3e-7 and the roundings).
__device__ __forceinline__ float erfc_pos(float t) {
  float u = fmaf(kErfA6, t, kErfA5);
  u = fmaf(u, t, kErfA4);
  u = fmaf(u, t, kErfA3);
  u = fmaf(u, t, kErfA2);
  u = fmaf(u, t, kErfA1);
  u *= t;
  u *= u + 2.0f;
  u *= u + 2.0f;
  u *= u + 2.0f;
  u *= u + 2.0f;
  return rcp_approx(1.0f + u);
}

// standard normal CDF Phi(p) = erfc(-p / sqrt 2) / 2: the tail half-erfc is
// taken directly for p < 0, so small values keep their relative accuracy
__device__ __forceinline__ float norm_cdf(float p) {
  const float h = 0.5f * erfc_pos(fabsf(p) * 0.70710678118654752440f);
  return p >= 0.0f ? 1.0f - h : h;
}
__device__ __forceinline__ float gelu_f(float p) { return p * norm_cdf(p); }
// GELU and its derivative from one evaluation of the normal CDF
__device__ __forceinline__ void gelu_and_grad_f(float p, float &g, float &dg) {
  const float cdf = norm_cdf(p);
  g = p * cdf;
  dg = cdf + p * 0.39894228040143267794f * expf(-0.5f * p * p);
}
__device__ __forceinline__ float gelu_grad_f(float p) {
  return norm_cdf(p) + p * 0.39894228040143267794f * expf(-0.5f * p * p);
}

// ---- packed float32 pairs (sm_100 f32x2 arithmetic) ------------------------
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 f2pack(float a, float b) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(f32x2 v, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ f32x2 f2fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 f2mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2add(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2splat(float c) { return f2pack(c, c); }

// GELU of two values at once, on packed pairs (the forward's activation):
// formula 7.1.28 with 1 / sqrt 2 folded into the coefficients (a_k 2^(-k/2))
// and q raised to the 16th power directly (four multiplies), then
// w = (p / 2) erfc(|p| / sqrt 2) and GELU(p) = p - w (p >= 0) or w (p < 0).
// The error of q^16 near p = 0 is scaled by p here: |GELU error| <= 4e-7
// max(1, |p|) in float32.
// (1 + a_1 t + ... + a_6 t^6)^16 of two |p| at once, the coefficients holding
// the 1 / sqrt 2 of erf(p / sqrt 2)
__device__ __forceinline__ void erf_q16(float a, float b, float &qa, float &qb) {
  const f32x2 t = f2pack(fabsf(a), fabsf(b));
  f32x2 q = f2fma(f2splat(5.38297490493278e-06f), t, f2splat(4.889063711743802e-05f));
  q = f2fma(q, t, f2splat(3.8003574445610866e-05f));
  q = f2fma(q, t, f2splat(0.0032776263542473316f));
  q = f2fma(q, t, f2splat(0.02114100567996502f));
  q = f2fma(q, t, f2splat(0.04986734688282013f));
  q = f2fma(q, t, f2splat(1.0f));
  q = f2mul(q, q);
  q = f2mul(q, q);
  q = f2mul(q, q);
  q = f2mul(q, q);
  f2unpack(q, qa, qb);
}

__device__ __forceinline__ void gelu2(float &a, float &b) {
  float qa, qb, wa, wb;
  erf_q16(a, b, qa, qb);
  f2unpack(f2mul(f2pack(rcp_approx(qa), rcp_approx(qb)), f2mul(f2pack(a, b), f2splat(0.5f))), wa,
           wb);
  a = a >= 0.0f ? a - wa : wa;
  b = b >= 0.0f ? b - wb : wb;
}

// 2 GELU of two values at once, for a caller that folds the 1/2 into its next
// multiply: w = p erfc(|p| / sqrt 2), 2 GELU(p) = 2 p - w (p >= 0) or w (p < 0);
// one multiply fewer than gelu2.
__device__ __forceinline__ void gelu2_dbl(float &a, float &b) {
  float qa, qb, wa, wb;
  erf_q16(a, b, qa, qb);
  f2unpack(f2mul(f2pack(rcp_approx(qa), rcp_approx(qb)), f2pack(a, b)), wa, wb);
  a = a >= 0.0f ? fmaf(2.0f, a, -wa) : wa;
  b = b >= 0.0f ? fmaf(2.0f, b, -wb) : wb;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// GELU'(p) = Phi(p) + p phi(p) of two values at once (the backward's dz), on
// packed pairs: Phi as erfc_pos (q - 1 carried through the squarings, 1 / sqrt 2
// folded into the coefficients), phi(p) = exp(-p^2 / 2) / sqrt(2 pi) as
// 2^(-p^2 log2(e) / 2).
__device__ __forceinline__ void gelu_grad2(float &a, float &b) {
  const f32x2 p = f2pack(a, b);
  const f32x2 t = f2pack(fabsf(a), fabsf(b));
  f32x2 u = f2fma(f2splat(5.38297490493278e-06f), t, f2splat(4.889063711743802e-05f));
  u = f2fma(u, t, f2splat(3.8003574445610866e-05f));
  u = f2fma(u, t, f2splat(0.0032776263542473316f));
  u = f2fma(u, t, f2splat(0.02114100567996502f));
  u = f2fma(u, t, f2splat(0.04986734688282013f));
  u = f2mul(u, t);
  u = f2mul(u, f2add(u, f2splat(2.0f)));
  u = f2mul(u, f2add(u, f2splat(2.0f)));
  u = f2mul(u, f2add(u, f2splat(2.0f)));
  u = f2mul(u, f2add(u, f2splat(2.0f)));
  float qa, qb;
  f2unpack(f2add(u, f2splat(1.0f)), qa, qb);
  float ha, hb;                                   // Phi(-|p|) = erfc(|p| / sqrt 2) / 2
  f2unpack(f2mul(f2pack(rcp_approx(qa), rcp_approx(qb)), f2splat(0.5f)), ha, hb);
  float ea, eb;                                   // -p^2 log2(e) / 2
  f2unpack(f2mul(f2mul(p, p), f2splat(-0.72134752044448170368f)), ea, eb);
  const f32x2 phi =
      f2mul(f2pack(ex2_approx(ea), ex2_approx(eb)), f2splat(0.39894228040143267794f));
  const f32x2 cdf = f2pack(a >= 0.0f ? 1.0f - ha : ha, b >= 0.0f ? 1.0f - hb : hb);
  f2unpack(f2fma(p, phi, cdf), a, b);
}

// weight c_k / N of last-axis mode k_l (1 on DC and Nyquist, else 2)
__device__ __forceinline__ float mode_weight(int k_l, int n_l, float inv_n) {
  bool edge = (k_l == 0) || ((n_l % 2 == 0) && (2 * k_l == n_l));
  return edge ? inv_n : 2.0f * inv_n;
}

}  // namespace fno
