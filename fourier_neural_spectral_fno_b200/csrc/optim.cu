// Optimiser step of the training loop: Adam on the float32 master weights
// fused with the copy of the updated weights in the storage dtype that the
// next forward reads (the precision-scheduling step of "Guaranteed
// approximation bounds and efficient mixed-precision training for neural
// operators", summary: training moves from mixed to full precision, so the
// copy's dtype follows the schedule).
//
// Adam is Kingma and Ba, "Adam: A Method for Stochastic Optimization",
// Algorithm 1, with the decoupled weight decay of Loshchilov and Hutter,
// "Decoupled Weight Decay Regularization":
//   g  = grad * grad_scale
//   m  = b1 m + (1 - b1) g            v = b2 v + (1 - b2) g^2
//   theta -= lr (m / bc1) / (sqrt(v / bc2) + eps) + lr wd theta
// with bc = 1 - b^t.  One pass over HBM: theta, m, v, g read once, theta, m,
// v and the storage copy written once (30 bytes per bf16 parameter).
#include <string.h>

#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int AT = 256;

__device__ __forceinline__ float adam_one(float th, float &m, float &v, float g,
                                          const AdamCoef &c) {
  g *= c.grad_scale;
  m = fmaf(c.beta1, m, c.one_minus_beta1 * g);
  v = fmaf(c.beta2, v, c.one_minus_beta2 * (g * g));
  const float den = sqrtf(v * c.inv_bc2) + c.eps;
  return th - c.lr * (m * c.inv_bc1) / den - c.lr_wd * th;
}

template <typename T> __device__ __forceinline__ void store4(T *p, float4 v);
template <> __device__ __forceinline__ void store4<float>(float *p, float4 v) {
  *reinterpret_cast<float4 *>(p) = v;
}
template <> __device__ __forceinline__ void store4<__half>(__half *p, float4 v) {
  __half2 lo = __floats2half2_rn(v.x, v.y), hi = __floats2half2_rn(v.z, v.w);
  uint2 u;
  memcpy(&u.x, &lo, 4);
  memcpy(&u.y, &hi, 4);
  *reinterpret_cast<uint2 *>(p) = u;
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *p, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  memcpy(&u.x, &lo, 4);
  memcpy(&u.y, &hi, 4);
  *reinterpret_cast<uint2 *>(p) = u;
}

// n4 groups of four through 16-byte accesses, then the n - 4 n4 tail
template <typename T>
__global__ void __launch_bounds__(AT)
    k_adam(long long n, long long n4, float *__restrict__ theta, float *__restrict__ m,
           float *__restrict__ v, const float *__restrict__ g, T *__restrict__ out, AdamCoef c) {
  const long long stride = (long long)gridDim.x * AT;
  for (long long i = (long long)blockIdx.x * AT + threadIdx.x; i < n4; i += stride) {
    float4 th = reinterpret_cast<const float4 *>(theta)[i];
    if (g) {
      float4 mm = reinterpret_cast<const float4 *>(m)[i];
      float4 vv = reinterpret_cast<const float4 *>(v)[i];
      const float4 gg = __ldg(reinterpret_cast<const float4 *>(g) + i);
      th.x = adam_one(th.x, mm.x, vv.x, gg.x, c);
      th.y = adam_one(th.y, mm.y, vv.y, gg.y, c);
      th.z = adam_one(th.z, mm.z, vv.z, gg.z, c);
      th.w = adam_one(th.w, mm.w, vv.w, gg.w, c);
      reinterpret_cast<float4 *>(theta)[i] = th;
      reinterpret_cast<float4 *>(m)[i] = mm;
      reinterpret_cast<float4 *>(v)[i] = vv;
    }
    if (out) store4<T>(out + 4 * i, th);
  }
  for (long long i = 4 * n4 + (long long)blockIdx.x * AT + threadIdx.x; i < n; i += stride) {
    float th = theta[i];
    if (g) {
      float mm = m[i], vv = v[i];
      th = adam_one(th, mm, vv, __ldg(g + i), c);
      theta[i] = th;
      m[i] = mm;
      v[i] = vv;
    }
    if (out) out[i] = from_f<T>(th);
  }
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
bool al8(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 7) == 0; }

template <typename T>
cudaError_t launch_adam_t(const Launch &L, long long n, float *theta, float *m, float *v,
                          const float *g, void *out, const AdamCoef &c) {
  // 16-byte groups need 16-byte aligned float arrays and an aligned 4-element copy
  const bool vec = al16(theta) && (!g || (al16(m) && al16(v) && al16(g))) &&
                   (!out || (sizeof(T) == 4 ? al16(out) : al8(out)));
  const long long n4 = vec ? n / 4 : 0;
  const long long work = n4 + (n - 4 * n4);
  long long blocks = (work + AT - 1) / AT;
  const long long cap = 8LL * L.num_sms;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  k_adam<T><<<(unsigned)blocks, AT, 0, L.stream>>>(n, n4, theta, m, v, g,
                                                   reinterpret_cast<T *>(out), c);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_adam(const Launch &L, long long n, float *theta, float *m, float *v,
                        const float *g, void *out, int out_dtype, const AdamCoef &c) {
  launch_begin(L);
  cudaError_t err;
  if (out_dtype == DT_F16) err = launch_adam_t<__half>(L, n, theta, m, v, g, out, c);
  else if (out_dtype == DT_BF16) err = launch_adam_t<__nv_bfloat16>(L, n, theta, m, v, g, out, c);
  else err = launch_adam_t<float>(L, n, theta, m, v, g, out, c);
  launch_end(L, g ? "adam" : "cast_params");
  return err;
}

}  // namespace fno
