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
__device__ __forceinline__ float gelu_f(float p) {
  return 0.5f * p * (1.0f + erff(p * 0.70710678118654752440f));
}
__device__ __forceinline__ float gelu_grad_f(float p) {
  return 0.5f * (1.0f + erff(p * 0.70710678118654752440f)) +
         p * 0.39894228040143267794f * expf(-0.5f * p * p);
}

// weight c_k / N of last-axis mode k_l (1 on DC and Nyquist, else 2)
__device__ __forceinline__ float mode_weight(int k_l, int n_l, float inv_n) {
  bool edge = (k_l == 0) || ((n_l % 2 == 0) && (2 * k_l == n_l));
  return edge ? inv_n : 2.0f * inv_n;
}

}  // namespace fno
