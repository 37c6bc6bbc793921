// Per-mode mixing (step S3) with CP-factorised spectral weights (TFNO,
// "Guaranteed approximation bounds and efficient mixed-precision training for
// neural operators", summary: factorised weights and a greedy ordering of the
// block's contractions):
//
//   R[i,o,k] = sum_r lam[r] A[i,r] B[o,r] C[k,r]
//   yhat[b,o,k] = (c_k / N) sum_r (lam[r] B[o,r]) C[k,r] sum_i xhat[b,i,k] A[i,r]
//
// The dense weight is never built.  The contraction runs in the order the
// greedy planner (contraction.py) chooses at low rank: xhat with A over i,
// then the elementwise product with C, then (lam B) over r.  One thread owns a
// (sample, mode) pair and holds its rank-r intermediate in registers; A and
// lam B are staged once per CTA in shared memory (every thread reads the same
// entries, so the reads are broadcasts).
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int CP_THREADS = 128;

template <typename T, int RMAX>
__global__ void __launch_bounds__(CP_THREADS)
    k_mix_cp(const float2 *__restrict__ xhat, const T *__restrict__ lam, const T *__restrict__ A,
             const T *__restrict__ Bf, const T *__restrict__ C, float2 *__restrict__ yhat,
             long long B, int Ci, int Co, long long K, int rank, int mL, int NL, float inv_n) {
  extern __shared__ __align__(16) unsigned char smem[];
  float2 *As = reinterpret_cast<float2 *>(smem);          // [Ci][RMAX]
  float2 *LBs = As + (size_t)Ci * RMAX;                    // [Co][RMAX]: lam[r] B[o, r]
  for (int e = threadIdx.x; e < Ci * RMAX; e += CP_THREADS) {
    const int i = e / RMAX, r = e - i * RMAX;
    As[e] = r < rank ? ldc<T>(A + 2 * ((long long)i * rank + r)) : make_float2(0.f, 0.f);
  }
  for (int e = threadIdx.x; e < Co * RMAX; e += CP_THREADS) {
    const int o = e / RMAX, r = e - o * RMAX;
    LBs[e] = r < rank ? cmul(ldc<T>(lam + 2 * r), ldc<T>(Bf + 2 * ((long long)o * rank + r)))
                      : make_float2(0.f, 0.f);
  }
  __syncthreads();
  const long long t = (long long)blockIdx.x * CP_THREADS + threadIdx.x;
  if (t >= B * K) return;
  const long long b = t / K, k = t - b * K;
  float2 f[RMAX];
#pragma unroll
  for (int r = 0; r < RMAX; ++r) f[r] = make_float2(0.f, 0.f);
  const float2 *xp = xhat + b * Ci * K + k;
  for (int i = 0; i < Ci; ++i) {
    const float2 xv = __ldg(xp + (long long)i * K);
    const float2 *ar = As + i * RMAX;
#pragma unroll
    for (int r = 0; r < RMAX; ++r) cfma(f[r], xv, ar[r]);
  }
#pragma unroll
  for (int r = 0; r < RMAX; ++r)
    f[r] = r < rank ? cmul(f[r], ldc<T>(C + 2 * (k * rank + r))) : make_float2(0.f, 0.f);
  const float w = mode_weight((int)(k % mL), NL, inv_n);
  float2 *yp = yhat + b * Co * K + k;
  for (int o = 0; o < Co; ++o) {
    float2 s = make_float2(0.f, 0.f);
    const float2 *lb = LBs + o * RMAX;
#pragma unroll
    for (int r = 0; r < RMAX; ++r) cfma(s, lb[r], f[r]);
    yp[(long long)o * K] = make_float2(w * s.x, w * s.y);
  }
}

template <typename T>
cudaError_t launch_cp_t(const Launch &L, const Geom &g, int Ci, int Co, int rank,
                        const float2 *xhat, const CpFactors &f, float2 *yhat) {
  const long long n = g.B * g.K;
  const unsigned grid = (unsigned)((n + CP_THREADS - 1) / CP_THREADS);
  auto go = [&](auto kern, int rmax) {
    const size_t smem = sizeof(float2) * (size_t)(Ci + Co) * rmax;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, CP_THREADS, smem, L.stream>>>(
        xhat, (const T *)f.lam, (const T *)f.A, (const T *)f.B, (const T *)f.C, yhat, g.B, Ci, Co,
        g.K, rank, g.mL, g.NL, g.inv_n);
    return cudaGetLastError();
  };
  if (rank <= 8) return go(k_mix_cp<T, 8>, 8);
  if (rank <= 16) return go(k_mix_cp<T, 16>, 16);
  return go(k_mix_cp<T, 32>, 32);
}

}  // namespace

cudaError_t launch_mix_cp(const Launch &L, const Geom &g, int dtype, int Ci, int Co, int rank,
                          const float2 *xhat, const CpFactors &f, float2 *yhat) {
  launch_begin(L);
  cudaError_t e;
  if (dtype == DT_F32) e = launch_cp_t<float>(L, g, Ci, Co, rank, xhat, f, yhat);
  else if (dtype == DT_F16) e = launch_cp_t<__half>(L, g, Ci, Co, rank, xhat, f, yhat);
  else e = launch_cp_t<__nv_bfloat16>(L, g, Ci, Co, rank, xhat, f, yhat);
  launch_end(L, "mix_cp");
  return e;
}

}  // namespace fno
