// Per-mode complex channel mixing (step S3) and its two adjoints on the CUDA
// cores (the tensor-core form for bfloat16 weights at 64 channels is in
// mix_tc.cu and is taken where it applies).
//
// For every kept mode k the block multiplies the batch of spectra
// xhat[:, :, k] (B x Ci) by the mode's weight matrix R[:, :, k] (Ci x Co).
// The weights are laid out [Ci][Co][K], so consecutive threads take
// consecutive modes and every load is coalesced; each thread keeps a register
// tile of the two free indices; the inverse transform's scale c_k / N is folded
// into the output here.
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int MX_THREADS = 128;   // consecutive modes per CTA (coalesced along k)

__device__ __forceinline__ float weight_of(long long k, int mL, int NL, float inv_n) {
  return mode_weight((int)(k % mL), NL, inv_n);
}

// Register tiles: a thread owns one mode k and a tile of the two free indices,
// so every value it loads feeds a whole row or column of complex multiply-adds
// (the tile sizes set how often each operand is re-read from L2).

// yhat[b,o,k] = w_k sum_i xhat[b,i,k] R[i,o,k]: tile OT output channels x BT
// batch entries, loop over i
template <typename T, int OT, int BT>
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_fwd(const float2 *__restrict__ xhat, const T *__restrict__ R, float2 *__restrict__ yhat,
              long long B, int Ci, int Co, long long K, int mL, int NL, float inv_n) {
  const long long k = (long long)blockIdx.x * MX_THREADS + threadIdx.x;
  const int o0 = blockIdx.y * OT;
  const long long b0 = (long long)blockIdx.z * BT;
  if (k >= K) return;
  float2 acc[OT][BT];
#pragma unroll
  for (int u = 0; u < OT; ++u)
#pragma unroll
    for (int v = 0; v < BT; ++v) acc[u][v] = make_float2(0.f, 0.f);
  const long long rstride = 2LL * Co * K;
  // small tiles unroll the reduction so several iterations' loads are in flight
  constexpr int UNR = OT * BT <= 8 ? 8 : 1;
#pragma unroll UNR
  for (int i = 0; i < Ci; ++i) {
    float2 r[OT], x[BT];
#pragma unroll
    for (int u = 0; u < OT; ++u)
      r[u] = o0 + u < Co ? ldc<T>(R + i * rstride + 2 * ((long long)(o0 + u) * K + k))
                         : make_float2(0.f, 0.f);
#pragma unroll
    for (int v = 0; v < BT; ++v)
      x[v] = b0 + v < B ? __ldg(xhat + ((b0 + v) * Ci + i) * K + k) : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < OT; ++u)
#pragma unroll
      for (int v = 0; v < BT; ++v) cfma(acc[u][v], x[v], r[u]);
  }
  const float w = weight_of(k, mL, NL, inv_n);
#pragma unroll
  for (int u = 0; u < OT; ++u)
#pragma unroll
    for (int v = 0; v < BT; ++v)
      if (o0 + u < Co && b0 + v < B)
        yhat[((b0 + v) * Co + o0 + u) * K + k] = make_float2(w * acc[u][v].x, w * acc[u][v].y);
}

// dR[i,o,k] = w_k sum_b conj(xhat[b,i,k]) D[b,o,k]: tile IT x OT, loop over b
template <int IT, int OT>
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_bwd_dr(const float2 *__restrict__ xhat, const float2 *__restrict__ D,
                 float *__restrict__ dR, long long B, int Ci, int Co, long long K, int mL, int NL,
                 float inv_n) {
  const long long k = (long long)blockIdx.x * MX_THREADS + threadIdx.x;
  const int o0 = blockIdx.y * OT, i0 = blockIdx.z * IT;
  if (k >= K) return;
  float2 acc[IT][OT];
#pragma unroll
  for (int u = 0; u < IT; ++u)
#pragma unroll
    for (int v = 0; v < OT; ++v) acc[u][v] = make_float2(0.f, 0.f);
  constexpr int UNR = IT * OT <= 8 ? 4 : 1;
#pragma unroll UNR
  for (long long b = 0; b < B; ++b) {
    float2 x[IT], d[OT];
#pragma unroll
    for (int u = 0; u < IT; ++u)
      x[u] = i0 + u < Ci ? __ldg(xhat + (b * Ci + i0 + u) * K + k) : make_float2(0.f, 0.f);
#pragma unroll
    for (int v = 0; v < OT; ++v)
      d[v] = o0 + v < Co ? __ldg(D + (b * Co + o0 + v) * K + k) : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < IT; ++u)
#pragma unroll
      for (int v = 0; v < OT; ++v) cfma_conj_a(acc[u][v], x[u], d[v]);
  }
  const float w = weight_of(k, mL, NL, inv_n);
#pragma unroll
  for (int u = 0; u < IT; ++u)
#pragma unroll
    for (int v = 0; v < OT; ++v)
      if (i0 + u < Ci && o0 + v < Co)
        reinterpret_cast<float2 *>(dR)[((long long)(i0 + u) * Co + o0 + v) * K + k] =
            make_float2(w * acc[u][v].x, w * acc[u][v].y);
}

// dxhat[b,i,k] = w_k sum_o D[b,o,k] conj(R[i,o,k]): tile IT input channels x BT
// batch entries, loop over o
template <typename T, int IT, int BT>
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_bwd_dx(const float2 *__restrict__ D, const T *__restrict__ R, float2 *__restrict__ dxhat,
                 long long B, int Ci, int Co, long long K, int mL, int NL, float inv_n) {
  const long long k = (long long)blockIdx.x * MX_THREADS + threadIdx.x;
  const int i0 = blockIdx.y * IT;
  const long long b0 = (long long)blockIdx.z * BT;
  if (k >= K) return;
  float2 acc[IT][BT];
#pragma unroll
  for (int u = 0; u < IT; ++u)
#pragma unroll
    for (int v = 0; v < BT; ++v) acc[u][v] = make_float2(0.f, 0.f);
  constexpr int UNR = IT * BT <= 8 ? 8 : 1;
#pragma unroll UNR
  for (int o = 0; o < Co; ++o) {
    float2 r[IT], d[BT];
#pragma unroll
    for (int u = 0; u < IT; ++u)
      r[u] = i0 + u < Ci ? ldc<T>(R + 2 * (((long long)(i0 + u) * Co + o) * K + k))
                         : make_float2(0.f, 0.f);
#pragma unroll
    for (int v = 0; v < BT; ++v)
      d[v] = b0 + v < B ? __ldg(D + ((b0 + v) * Co + o) * K + k) : make_float2(0.f, 0.f);
#pragma unroll
    for (int u = 0; u < IT; ++u)
#pragma unroll
      for (int v = 0; v < BT; ++v) cfma_conj_b(acc[u][v], d[v], r[u]);
  }
  const float w = weight_of(k, mL, NL, inv_n);
#pragma unroll
  for (int u = 0; u < IT; ++u)
#pragma unroll
    for (int v = 0; v < BT; ++v)
      if (i0 + u < Ci && b0 + v < B)
        dxhat[((b0 + v) * Ci + i0 + u) * K + k] = make_float2(w * acc[u][v].x, w * acc[u][v].y);
}

constexpr int MX_BT = 4;  // batch entries per thread of the small-shape kernels

// small shapes: thread per (mode, o), MX_BT batch entries (more threads)
template <typename T>
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_fwd_1(const float2 *__restrict__ xhat, const T *__restrict__ R, float2 *__restrict__ yhat,
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

// small shapes: thread per (mode, o, i), loop over b
// dR[i,o,k] = sum_b conj(xhat[b,i,k]) * w_k D[b,o,k]
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_bwd_dr_1(const float2 *__restrict__ xhat, const float2 *__restrict__ D,
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

// small shapes: thread per (mode, i), MX_BT batch entries
// dxhat[b,i,k] = sum_o w_k D[b,o,k] conj(R[i,o,k])
template <typename T>
__global__ void __launch_bounds__(MX_THREADS)
    k_mix_bwd_dx_1(const float2 *__restrict__ D, const T *__restrict__ R, float2 *__restrict__ dxhat,
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

// the tiled kernels (4 x 8) where they still leave about eight warps per SM,
// else the one-channel kernels (measured faster at the small shapes)
inline bool big_tiles(long long K, long long n_a, long long n_b, int num_sms) {
  const long long threads = ((K + MX_THREADS - 1) / MX_THREADS) * MX_THREADS *
                            ((n_a + 3) / 4) * ((n_b + 7) / 8);
  return threads >= (long long)num_sms * 32 * 8;
}

template <typename T, int OT, int BT>
cudaError_t mix_fwd_t(const Launch &L, const Geom &g, int Ci, int Co, const float2 *xhat,
                      const void *R, float2 *yhat) {
  dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)((Co + OT - 1) / OT),
            (unsigned)((g.B + BT - 1) / BT));
  k_mix_fwd<T, OT, BT><<<grid, MX_THREADS, 0, L.stream>>>(xhat, (const T *)R, yhat, g.B, Ci, Co,
                                                          g.K, g.mL, g.NL, g.inv_n);
  return cudaGetLastError();
}

template <typename T, int IT, int BT>
cudaError_t mix_dx_t(const Launch &L, const Geom &g, int Ci, int Co, const float2 *D,
                     const void *R, float2 *dxhat) {
  dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)((Ci + IT - 1) / IT),
            (unsigned)((g.B + BT - 1) / BT));
  k_mix_bwd_dx<T, IT, BT><<<grid, MX_THREADS, 0, L.stream>>>(D, (const T *)R, dxhat, g.B, Ci, Co,
                                                             g.K, g.mL, g.NL, g.inv_n);
  return cudaGetLastError();
}

template <typename T>
cudaError_t mix_fwd_small(const Launch &L, const Geom &g, int Ci, int Co, const float2 *xhat,
                          const void *R, float2 *yhat) {
  dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)Co,
            (unsigned)((g.B + MX_BT - 1) / MX_BT));
  k_mix_fwd_1<T><<<grid, MX_THREADS, 0, L.stream>>>(xhat, (const T *)R, yhat, g.B, Ci, Co, g.K,
                                                    g.mL, g.NL, g.inv_n);
  return cudaGetLastError();
}

template <typename T>
cudaError_t mix_dx_small(const Launch &L, const Geom &g, int Ci, int Co, const float2 *D,
                         const void *R, float2 *dxhat) {
  dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)Ci,
            (unsigned)((g.B + MX_BT - 1) / MX_BT));
  k_mix_bwd_dx_1<T><<<grid, MX_THREADS, 0, L.stream>>>(D, (const T *)R, dxhat, g.B, Ci, Co, g.K,
                                                       g.mL, g.NL, g.inv_n);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mix_fwd(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                           const float2 *xhat, const void *R, float2 *yhat) {
  const bool big = big_tiles(g.K, Co, g.B, L.num_sms);
  const bool tc = L.tc != 0 && L.tc != 2 && mix_tc_supported(g, dtype, false, Ci, Co, xhat, R, yhat);
  launch_begin(L);
  cudaError_t e;
  if (tc)
    e = launch_mix_tc(L, g, false, Ci, Co, xhat, R, yhat);
  else if (dtype == DT_F32)
    e = big ? mix_fwd_t<float, 4, 8>(L, g, Ci, Co, xhat, R, yhat)
            : mix_fwd_small<float>(L, g, Ci, Co, xhat, R, yhat);
  else if (dtype == DT_F16)
    e = big ? mix_fwd_t<__half, 4, 8>(L, g, Ci, Co, xhat, R, yhat)
            : mix_fwd_small<__half>(L, g, Ci, Co, xhat, R, yhat);
  else
    e = big ? mix_fwd_t<__nv_bfloat16, 4, 8>(L, g, Ci, Co, xhat, R, yhat)
            : mix_fwd_small<__nv_bfloat16>(L, g, Ci, Co, xhat, R, yhat);
  launch_end(L, tc ? "mix_fwd_tc" : "mix_fwd");
  return e;
}

cudaError_t launch_mix_bwd_dr(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                              const float2 *xhat, const float2 *D, float *dR) {
  const bool big = big_tiles(g.K, Ci, Co * 2, L.num_sms);
  const bool tc = L.tc != 0 && L.tc != 2 && mix_tc_dr_supported(g, dtype, Ci, Co, xhat, D, dR);
  launch_begin(L);
  if (tc) {
    const cudaError_t e = launch_mix_tc_dr(L, g, Co, xhat, D, dR);
    launch_end(L, "mix_bwd_dr_tc");
    return e;
  }
  if (big) {
    dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)((Co + 3) / 4),
              (unsigned)((Ci + 3) / 4));
    k_mix_bwd_dr<4, 4><<<grid, MX_THREADS, 0, L.stream>>>(xhat, D, dR, g.B, Ci, Co, g.K, g.mL,
                                                          g.NL, g.inv_n);
  } else {
    dim3 grid((unsigned)((g.K + MX_THREADS - 1) / MX_THREADS), (unsigned)Co, (unsigned)Ci);
    k_mix_bwd_dr_1<<<grid, MX_THREADS, 0, L.stream>>>(xhat, D, dR, g.B, Ci, Co, g.K, g.mL, g.NL,
                                                       g.inv_n);
  }
  launch_end(L, "mix_bwd_dr");
  return cudaGetLastError();
}

cudaError_t launch_mix_bwd_dx(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                              const float2 *D, const void *R, float2 *dxhat) {
  const bool big = big_tiles(g.K, Ci, g.B, L.num_sms);
  const bool tc = L.tc != 0 && L.tc != 2 && mix_tc_supported(g, dtype, true, Ci, Co, D, R, dxhat);
  launch_begin(L);
  cudaError_t e;
  if (tc)
    e = launch_mix_tc(L, g, true, Ci, Co, D, R, dxhat);
  else if (dtype == DT_F32)
    e = big ? mix_dx_t<float, 4, 8>(L, g, Ci, Co, D, R, dxhat)
            : mix_dx_small<float>(L, g, Ci, Co, D, R, dxhat);
  else if (dtype == DT_F16)
    e = big ? mix_dx_t<__half, 4, 8>(L, g, Ci, Co, D, R, dxhat)
            : mix_dx_small<__half>(L, g, Ci, Co, D, R, dxhat);
  else
    e = big ? mix_dx_t<__nv_bfloat16, 4, 8>(L, g, Ci, Co, D, R, dxhat)
            : mix_dx_small<__nv_bfloat16>(L, g, Ci, Co, D, R, dxhat);
  launch_end(L, tc ? "mix_bwd_dx_tc" : "mix_bwd_dx");
  return e;
}

}  // namespace fno
