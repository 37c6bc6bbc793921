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

// ---------------------------------------------------------------------------
// backward through the factors
// ---------------------------------------------------------------------------
namespace fno {

namespace {

// the dense weight R[i,o,k] = sum_r lam[r] A[i,r] B[o,r] C[k,r], rounded to
// the storage dtype (the dense backward's dxhat reads it)
template <typename T>
__global__ void __launch_bounds__(256)
    k_cp_rebuild(const T *__restrict__ lam, const T *__restrict__ A, const T *__restrict__ Bf,
                 const T *__restrict__ C, T *__restrict__ R, int Ci, int Co, long long K,
                 int rank) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)Ci * Co * K) return;
  const long long k = t % K, io = t / K;
  const int o = (int)(io % Co), i = (int)(io / Co);
  float2 s = make_float2(0.f, 0.f);
  for (int r = 0; r < rank; ++r) {
    const float2 la = cmul(ldc<T>(lam + 2 * r), ldc<T>(A + 2 * ((long long)i * rank + r)));
    const float2 bc = cmul(ldc<T>(Bf + 2 * ((long long)o * rank + r)),
                           ldc<T>(C + 2 * (k * rank + r)));
    cfma(s, la, bc);
  }
  R[2 * t] = from_f<T>(s.x);
  R[2 * t + 1] = from_f<T>(s.y);
}

// S_m[n][r] = sum over the two other weight axes of dR conj(product of their
// factors): m = 0 (n = i: sum over o, k of dR conj(B C)), 1 (n = o: over i, k
// of dR conj(A C)), 2 (n = k: over i, o of dR conj(A B)).  One CTA per n;
// every thread keeps all rank sums of its share, then a shared-memory tree.
template <typename T>
__global__ void __launch_bounds__(256)
    k_cp_project(const float2 *__restrict__ dR, const T *__restrict__ A,
                 const T *__restrict__ Bf, const T *__restrict__ C, float2 *__restrict__ S,
                 int m, int Ci, int Co, long long K, int rank) {
  __shared__ float2 red[256];
  const int n = blockIdx.x;
  const long long other = m == 0 ? (long long)Co * K : m == 1 ? (long long)Ci * K : (long long)Ci * Co;
  float2 acc[kMaxCpRank];
#pragma unroll
  for (int r = 0; r < kMaxCpRank; ++r) acc[r] = make_float2(0.f, 0.f);
  for (long long e = threadIdx.x; e < other; e += blockDim.x) {
    long long i, o, k;
    const T *f1, *f2;
    if (m == 0) { i = n; o = e / K; k = e % K; f1 = Bf + 2 * o * rank; f2 = C + 2 * k * rank; }
    else if (m == 1) { o = n; i = e / K; k = e % K; f1 = A + 2 * i * rank; f2 = C + 2 * k * rank; }
    else { k = n; i = e / Co; o = e % Co; f1 = A + 2 * i * rank; f2 = Bf + 2 * o * rank; }
    const float2 d = __ldg(dR + (i * Co + o) * K + k);
#pragma unroll
    for (int r = 0; r < kMaxCpRank; ++r)
      if (r < rank) cfma_conj_b(acc[r], d, cmul(ldc<T>(f1 + 2 * r), ldc<T>(f2 + 2 * r)));
  }
#pragma unroll
  for (int r = 0; r < kMaxCpRank; ++r) {
    if (r >= rank) break;                    // uniform across the CTA
    red[threadIdx.x] = acc[r];
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if ((int)threadIdx.x < w) {
        red[threadIdx.x].x += red[threadIdx.x + w].x;
        red[threadIdx.x].y += red[threadIdx.x + w].y;
      }
      __syncthreads();
    }
    if (threadIdx.x == 0) S[(long long)n * rank + r] = red[0];
    __syncthreads();
  }
}

// dA = conj(lam) S_A, dB = conj(lam) S_B, dC = conj(lam) S_C (in place into the
// outputs) and dlam[r] = sum_i conj(A[i,r]) S_A[i,r]
template <typename T>
__global__ void __launch_bounds__(256)
    k_cp_finish(const T *__restrict__ lam, const T *__restrict__ A, const float2 *__restrict__ SA,
                float2 *__restrict__ dA, float2 *__restrict__ dB, float2 *__restrict__ dC,
                float2 *__restrict__ dlam, int Ci, int Co, long long K, int rank) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nA = (long long)Ci * rank, nB = (long long)Co * rank, nC = K * rank;
  if (t < nA) {
    const float2 l = ldc<T>(lam + 2 * (t % rank));
    const float2 s = SA[t];
    dA[t] = make_float2(l.x * s.x + l.y * s.y, l.x * s.y - l.y * s.x);   // conj(l) s
  } else if (t < nA + nB) {
    const long long u = t - nA;
    const float2 l = ldc<T>(lam + 2 * (u % rank)), s = dB[u];
    dB[u] = make_float2(l.x * s.x + l.y * s.y, l.x * s.y - l.y * s.x);
  } else if (t < nA + nB + nC) {
    const long long u = t - nA - nB;
    const float2 l = ldc<T>(lam + 2 * (u % rank)), s = dC[u];
    dC[u] = make_float2(l.x * s.x + l.y * s.y, l.x * s.y - l.y * s.x);
  } else if (t < nA + nB + nC + rank) {
    const int r = (int)(t - nA - nB - nC);
    float2 s = make_float2(0.f, 0.f);
    for (int i = 0; i < Ci; ++i) cfma_conj_a(s, ldc<T>(A + 2 * ((long long)i * rank + r)),
                                             SA[(long long)i * rank + r]);
    dlam[r] = s;
  }
}

template <typename T>
cudaError_t cp_rebuild_t(const Launch &L, const Geom &g, int Ci, int Co, int rank,
                         const CpFactors &f, void *R) {
  const long long n = (long long)Ci * Co * g.K;
  k_cp_rebuild<T><<<(unsigned)((n + 255) / 256), 256, 0, L.stream>>>(
      (const T *)f.lam, (const T *)f.A, (const T *)f.B, (const T *)f.C, (T *)R, Ci, Co, g.K, rank);
  return cudaGetLastError();
}

template <typename T>
cudaError_t cp_grads_t(const Launch &L, const Geom &g, int Ci, int Co, int rank,
                       const CpFactors &f, const float *dR, float *SA, float *dlam, float *dA,
                       float *dB, float *dC) {
  const float2 *d = reinterpret_cast<const float2 *>(dR);
  launch_begin(L);
  k_cp_project<T><<<Ci, 256, 0, L.stream>>>(d, (const T *)f.A, (const T *)f.B, (const T *)f.C,
                                            reinterpret_cast<float2 *>(SA), 0, Ci, Co, g.K, rank);
  launch_end(L, "cp_project");
  launch_begin(L);
  k_cp_project<T><<<Co, 256, 0, L.stream>>>(d, (const T *)f.A, (const T *)f.B, (const T *)f.C,
                                            reinterpret_cast<float2 *>(dB), 1, Ci, Co, g.K, rank);
  launch_end(L, "cp_project");
  launch_begin(L);
  k_cp_project<T><<<(unsigned)g.K, 256, 0, L.stream>>>(
      d, (const T *)f.A, (const T *)f.B, (const T *)f.C, reinterpret_cast<float2 *>(dC), 2, Ci, Co,
      g.K, rank);
  launch_end(L, "cp_project");
  const long long n = ((long long)Ci + Co + g.K) * rank + rank;
  launch_begin(L);
  k_cp_finish<T><<<(unsigned)((n + 255) / 256), 256, 0, L.stream>>>(
      (const T *)f.lam, (const T *)f.A, reinterpret_cast<const float2 *>(SA),
      reinterpret_cast<float2 *>(dA), reinterpret_cast<float2 *>(dB),
      reinterpret_cast<float2 *>(dC), reinterpret_cast<float2 *>(dlam), Ci, Co, g.K, rank);
  launch_end(L, "cp_finish");
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cp_rebuild(const Launch &L, const Geom &g, int dtype, int Ci, int Co, int rank,
                              const CpFactors &f, void *R) {
  launch_begin(L);
  cudaError_t e = dtype == DT_F32   ? cp_rebuild_t<float>(L, g, Ci, Co, rank, f, R)
                  : dtype == DT_F16 ? cp_rebuild_t<__half>(L, g, Ci, Co, rank, f, R)
                                    : cp_rebuild_t<__nv_bfloat16>(L, g, Ci, Co, rank, f, R);
  launch_end(L, "cp_rebuild");
  return e;
}

cudaError_t launch_cp_grads(const Launch &L, const Geom &g, int dtype, int Ci, int Co, int rank,
                            const CpFactors &f, const float *dR, float *scratch, float *dlam,
                            float *dA, float *dB, float *dC) {
  if (dtype == DT_F32) return cp_grads_t<float>(L, g, Ci, Co, rank, f, dR, scratch, dlam, dA, dB, dC);
  if (dtype == DT_F16) return cp_grads_t<__half>(L, g, Ci, Co, rank, f, dR, scratch, dlam, dA, dB, dC);
  return cp_grads_t<__nv_bfloat16>(L, g, Ci, Co, rank, f, dR, scratch, dlam, dA, dB, dC);
}

}  // namespace fno
