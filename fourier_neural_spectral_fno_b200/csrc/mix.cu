// Per-mode complex channel mixing (step S3) and its two adjoints.
//
// For every kept mode k the block multiplies the batch of spectra
// xhat[:, :, k] (B x Ci) by the mode's weight matrix R[:, :, k] (Ci x Co).
// The weights are laid out [Ci][Co][K], so consecutive threads take
// consecutive modes and every weight load is coalesced; the inverse
// transform's scale c_k / N is folded into the output here.
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int MX_THREADS = 128;
constexpr int MX_BT = 4;  // batch entries per thread

__device__ __forceinline__ float weight_of(long long k, int mL, int NL, float inv_n) {
  return mode_weight((int)(k % mL), NL, inv_n);
}

template <typename T>
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_fwd(const float2 *__restrict__ xhat, const T *__restrict__ R, float2 *__restrict__ yhat,
              long long B, int Ci, int Co, long long K, int mL, int NL, float inv_n) {
  const long long k = (long long)blockIdx.x * MX_THREADS + threadIdx.x;
  const int o = blockIdx.y;
  const long long b0 = (long long)blockIdx.z * MX_BT;
  if (k >= K) return;
  float2 acc[MX_BT];
#pragma unroll
  for (int j = 0; j < MX_BT; ++j) acc[j] = make_float2(0.f, 0.f);
  const T *rp = R + 2 * ((long long)o * K + k);
  const long long rstride = 2LL * Co * K;
  const float2 *xp = xhat + b0 * Ci * K + k;
#pragma unroll 8
  for (int i = 0; i < Ci; ++i) {
    const float2 r = ldc<T>(rp + i * rstride);
#pragma unroll
    for (int j = 0; j < MX_BT; ++j)
      if (b0 + j < B) cfma(acc[j], __ldg(xp + (j * Ci + i) * K), r);
  }
  const float w = weight_of(k, mL, NL, inv_n);
#pragma unroll
  for (int j = 0; j < MX_BT; ++j)
    if (b0 + j < B) yhat[((b0 + j) * Co + o) * K + k] = make_float2(w * acc[j].x, w * acc[j].y);
}

// dR[i,o,k] = sum_b conj(xhat[b,i,k]) * w_k D[b,o,k]
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_bwd_dr(const float2 *__restrict__ xhat, const float2 *__restrict__ D,
                 float *__restrict__ dR, long long B, int Ci, int Co, long long K, int mL, int NL,
                 float inv_n) {
  const long long k = (long long)blockIdx.x * MX_THREADS + threadIdx.x;
  const int o = blockIdx.y, i = blockIdx.z;
  if (k >= K) return;
  float2 s = make_float2(0.f, 0.f);
  for (long long b = 0; b < B; ++b)
    cfma_conj_a(s, __ldg(xhat + (b * Ci + i) * K + k), __ldg(D + (b * Co + o) * K + k));
  const float w = weight_of(k, mL, NL, inv_n);
  reinterpret_cast<float2 *>(dR)[((long long)i * Co + o) * K + k] = make_float2(w * s.x, w * s.y);
}

// dxhat[b,i,k] = sum_o w_k D[b,o,k] conj(R[i,o,k])
template <typename T>
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_bwd_dx(const float2 *__restrict__ D, const T *__restrict__ R, float2 *__restrict__ dxhat,
                 long long B, int Ci, int Co, long long K, int mL, int NL, float inv_n) {
  const long long k = (long long)blockIdx.x * MX_THREADS + threadIdx.x;
  const int i = blockIdx.y;
  const long long b0 = (long long)blockIdx.z * MX_BT;
  if (k >= K) return;
  float2 acc[MX_BT];
#pragma unroll
  for (int j = 0; j < MX_BT; ++j) acc[j] = make_float2(0.f, 0.f);
  for (int o = 0; o < Co; ++o) {
    const float2 r = ldc<T>(R + 2 * (((long long)i * Co + o) * K + k));
#pragma unroll
    for (int j = 0; j < MX_BT; ++j)
      if (b0 + j < B) cfma_conj_b(acc[j], __ldg(D + ((b0 + j) * Co + o) * K + k), r);
  }
  const float w = weight_of(k, mL, NL, inv_n);
#pragma unroll
  for (int j = 0; j < MX_BT; ++j)
    if (b0 + j < B) dxhat[((b0 + j) * Ci + i) * K + k] = make_float2(w * acc[j].x, w * acc[j].y);
}

}  // namespace

cudaError_t launch_mix_fwd(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                           const float2 *xhat, const void *R, float2 *yhat) {
  dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)Co,
            (unsigned)((g.B + MX_BT - 1) / MX_BT));
  launch_begin(L);
  if (dtype == DT_F32)
    k_mix_fwd<float><<<grid, MX_THREADS, 0, L.stream>>>(
        xhat, (const float *)R, yhat, g.B, Ci, Co, g.K, g.mL, g.NL, g.inv_n);
  else if (dtype == DT_F16)
    k_mix_fwd<__half><<<grid, MX_THREADS, 0, L.stream>>>(
        xhat, (const __half *)R, yhat, g.B, Ci, Co, g.K, g.mL, g.NL, g.inv_n);
  else
    k_mix_fwd<__nv_bfloat16><<<grid, MX_THREADS, 0, L.stream>>>(
        xhat, (const __nv_bfloat16 *)R, yhat, g.B, Ci, Co, g.K, g.mL, g.NL, g.inv_n);
  launch_end(L, "mix_fwd");
  return cudaGetLastError();
}

cudaError_t launch_mix_bwd_dr(const Launch &L, const Geom &g, int Ci, int Co, const float2 *xhat,
                              const float2 *D, float *dR) {
  dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)Co, (unsigned)Ci);
  launch_begin(L);
  k_mix_bwd_dr<<<grid, MX_THREADS, 0, L.stream>>>(xhat, D, dR, g.B, Ci, Co, g.K, g.mL, g.NL,
                                                  g.inv_n);
  launch_end(L, "mix_bwd_dr");
  return cudaGetLastError();
}

cudaError_t launch_mix_bwd_dx(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                              const float2 *D, const void *R, float2 *dxhat) {
  dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)Ci,
            (unsigned)((g.B + MX_BT - 1) / MX_BT));
  launch_begin(L);
  if (dtype == DT_F32)
    k_mix_bwd_dx<float><<<grid, MX_THREADS, 0, L.stream>>>(
        D, (const float *)R, dxhat, g.B, Ci, Co, g.K, g.mL, g.NL, g.inv_n);
  else if (dtype == DT_F16)
    k_mix_bwd_dx<__half><<<grid, MX_THREADS, 0, L.stream>>>(
        D, (const __half *)R, dxhat, g.B, Ci, Co, g.K, g.mL, g.NL, g.inv_n);
  else
    k_mix_bwd_dx<__nv_bfloat16><<<grid, MX_THREADS, 0, L.stream>>>(
        D, (const __nv_bfloat16 *)R, dxhat, g.B, Ci, Co, g.K, g.mL, g.NL, g.inv_n);
  launch_end(L, "mix_bwd_dx");
  return cudaGetLastError();
}

}  // namespace fno
