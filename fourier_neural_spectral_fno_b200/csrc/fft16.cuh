// Sixteen-point complex DFT in registers (radix 4 x 4), the building block of
// the pruned transforms in transform_fft.cu and spec_mid.cu.
//
//   fft16<-1>(z): z[m] <- sum_a z[a] exp(-2 pi i m a / 16)   (forward)
//   fft16<+1>(z): z[m] <- sum_a z[a] exp(+2 pi i m a / 16)   (inverse, unscaled)
//
// With a = 4 a1 + a0 and m = m0 + 4 m1 the sum splits into four 4-point DFTs
// over a1, the twiddles exp(SIGN 2 pi i a0 m0 / 16), and four 4-point DFTs
// over a0 (Cooley and Tukey, "An algorithm for the machine calculation of
// complex Fourier series", 1965).  All indices are compile-time constants,
// so the arrays stay in registers.
#pragma once

#include <cuda_runtime.h>

namespace fno {
namespace fft {

// cos and sin of pi e / 8, e = 0..9
__device__ __forceinline__ float cospi8(int e) {
  constexpr float c[10] = {1.0f,         0.92387953f, 0.70710678f, 0.38268343f, 0.0f,
                           -0.38268343f, -0.70710678f, -0.92387953f, -1.0f,     -0.92387953f};
  return c[e];
}
__device__ __forceinline__ float sinpi8(int e) {
  constexpr float s[10] = {0.0f,        0.38268343f, 0.70710678f, 0.92387953f, 1.0f,
                           0.92387953f, 0.70710678f, 0.38268343f, 0.0f,        -0.38268343f};
  return s[e];
}

// 4-point DFT with kernel exp(SIGN 2 pi i / 4) = SIGN i
template <int SIGN>
__device__ __forceinline__ void dft4(float2 x0, float2 x1, float2 x2, float2 x3, float2 &y0,
                                     float2 &y1, float2 &y2, float2 &y3) {
  const float2 s02 = make_float2(x0.x + x2.x, x0.y + x2.y);
  const float2 d02 = make_float2(x0.x - x2.x, x0.y - x2.y);
  const float2 s13 = make_float2(x1.x + x3.x, x1.y + x3.y);
  const float2 d13 = make_float2(x1.x - x3.x, x1.y - x3.y);
  y0 = make_float2(s02.x + s13.x, s02.y + s13.y);
  y2 = make_float2(s02.x - s13.x, s02.y - s13.y);
  // SIGN i d13 = (-SIGN d13.y, SIGN d13.x)
  if (SIGN < 0) {
    y1 = make_float2(d02.x + d13.y, d02.y - d13.x);
    y3 = make_float2(d02.x - d13.y, d02.y + d13.x);
  } else {
    y1 = make_float2(d02.x - d13.y, d02.y + d13.x);
    y3 = make_float2(d02.x + d13.y, d02.y - d13.x);
  }
}

// z * exp(SIGN i pi e / 8)
template <int SIGN>
__device__ __forceinline__ float2 twiddle(float2 z, int e) {
  if (e == 0) return z;
  if (e == 4) return SIGN < 0 ? make_float2(z.y, -z.x) : make_float2(-z.y, z.x);
  const float c = cospi8(e), s = SIGN < 0 ? -sinpi8(e) : sinpi8(e);
  return make_float2(fmaf(z.x, c, -z.y * s), fmaf(z.x, s, z.y * c));
}

template <int SIGN>
__device__ __forceinline__ void fft16(float2 (&z)[16]) {
  float2 t[4][4];
#pragma unroll
  for (int a0 = 0; a0 < 4; ++a0)
    dft4<SIGN>(z[a0], z[4 + a0], z[8 + a0], z[12 + a0], t[a0][0], t[a0][1], t[a0][2], t[a0][3]);
#pragma unroll
  for (int a0 = 1; a0 < 4; ++a0)
#pragma unroll
    for (int m0 = 1; m0 < 4; ++m0) t[a0][m0] = twiddle<SIGN>(t[a0][m0], a0 * m0);
#pragma unroll
  for (int m0 = 0; m0 < 4; ++m0)
    dft4<SIGN>(t[0][m0], t[1][m0], t[2][m0], t[3][m0], z[m0], z[m0 + 4], z[m0 + 8], z[m0 + 12]);
}

}  // namespace fft
}  // namespace fno
