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
// erf(t) for t >= 0: Chebyshev least-squares fit on [0, 3.9] evaluated by
// Horner's rule in x = (t - 1.95) / 1.95; 1 beyond 3.9 (1 - erf(3.9) = 3.5e-8).
// Coefficients from fourier_neural_spectral_fno_b200/gen_erf_poly.py; the
// float32 evaluation is within 6e-7 of erf (tests/test_gelu_poly.py).  It has
// no branches, so the GELUs of a thread's channels interleave freely.
__device__ __forceinline__ float erf_pos(float t) {
  const float x = (fminf(t, 3.9f) - 1.95f) * 0.51282054f;
  float a = 0.0026791077f;
  a = fmaf(a, x, -0.0049660155f);
  a = fmaf(a, x, -0.013497429f);
  a = fmaf(a, x, 0.03540305f);
  a = fmaf(a, x, 0.015209468f);
  a = fmaf(a, x, -0.10800477f);
  a = fmaf(a, x, 0.063275486f);
  a = fmaf(a, x, 0.14825702f);
  a = fmaf(a, x, -0.25860572f);
  a = fmaf(a, x, 0.04010987f);
  a = fmaf(a, x, 0.33213925f);
  a = fmaf(a, x, -0.4308476f);
  a = fmaf(a, x, 0.096189916f);
  a = fmaf(a, x, 0.3598901f);
  a = fmaf(a, x, -0.5448647f);
  a = fmaf(a, x, 0.4110579f);
  a = fmaf(a, x, -0.18670471f);
  a = fmaf(a, x, 0.04910043f);
  a = fmaf(a, x, 0.9941793f);
  return t > 3.9f ? 1.0f : a;
}

// standard normal CDF Phi(p) = (1 + erf(p / sqrt 2)) / 2
__device__ __forceinline__ float norm_cdf(float p) {
  const float e = erf_pos(fabsf(p) * 0.70710678118654752440f);
  return 0.5f + 0.5f * copysignf(e, p);
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

// GELU of two values at once: the erf polynomial of erf_pos on packed pairs.
// |p| is clamped at 3.9 sqrt(2) (erf(3.9) = 1 - 3.5e-8) and the variable change
// x = |p| / (1.95 sqrt 2) - 1 is one fused multiply-add.
__device__ __forceinline__ void gelu2(float &a, float &b) {
  const float ta = fminf(fabsf(a), 5.5154328f), tb = fminf(fabsf(b), 5.5154328f);
  const f32x2 x = f2fma(f2pack(ta, tb), f2splat(0.36261886f), f2splat(-1.0f));
  f32x2 e = f2splat(0.0026791077f);
  e = f2fma(e, x, f2splat(-0.0049660155f));
  e = f2fma(e, x, f2splat(-0.013497429f));
  e = f2fma(e, x, f2splat(0.03540305f));
  e = f2fma(e, x, f2splat(0.015209468f));
  e = f2fma(e, x, f2splat(-0.10800477f));
  e = f2fma(e, x, f2splat(0.063275486f));
  e = f2fma(e, x, f2splat(0.14825702f));
  e = f2fma(e, x, f2splat(-0.25860572f));
  e = f2fma(e, x, f2splat(0.04010987f));
  e = f2fma(e, x, f2splat(0.33213925f));
  e = f2fma(e, x, f2splat(-0.4308476f));
  e = f2fma(e, x, f2splat(0.096189916f));
  e = f2fma(e, x, f2splat(0.3598901f));
  e = f2fma(e, x, f2splat(-0.5448647f));
  e = f2fma(e, x, f2splat(0.4110579f));
  e = f2fma(e, x, f2splat(-0.18670471f));
  e = f2fma(e, x, f2splat(0.04910043f));
  e = f2fma(e, x, f2splat(0.9941793f));
  float ea, eb;
  f2unpack(e, ea, eb);
  const f32x2 phi = f2fma(f2pack(copysignf(ea, a), copysignf(eb, b)), f2splat(0.5f), f2splat(0.5f));
  f2unpack(f2mul(phi, f2pack(a, b)), a, b);
}

// weight c_k / N of last-axis mode k_l (1 on DC and Nyquist, else 2)
__device__ __forceinline__ float mode_weight(int k_l, int n_l, float inv_n) {
  bool edge = (k_l == 0) || ((n_l % 2 == 0) && (2 * k_l == n_l));
  return edge ? inv_n : 2.0f * inv_n;
}

}  // namespace fno
