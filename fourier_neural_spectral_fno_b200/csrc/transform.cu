// Truncated forward transform of the FNO block (steps S0-S2) and the inverse
// of the outer axis for 3D grids.
//
// S1 (last axis) is a dense contraction of each row of N_L points with the
// [N_L x m_L] matrix exp(-2 pi i k n / N_L); S2 contracts the resulting rows
// along the slab axis with the kept wavenumbers of that axis.  Both run in one
// kernel per (plane, band of rows): the plane's rows are streamed through
// shared memory once, so x is read from HBM exactly once.  Bands write
// partial spectra that the finishing kernel sums (and, for 3D grids,
// contracts along the outer axis).
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int FS_THREADS = 256;
constexpr int FS_RT = 64;   // rows per tile
constexpr int FS_NC = 64;   // columns per chunk
constexpr int FS_MAXJ = 4;  // last-axis modes per thread column (m_L <= 64)

struct FwdSlabArgs {
  const void *in0, *in1;
  float2 *zpart;           // [nbands][planes][QS][mL]
  long long planes;
  int S, NL, mL, mS, QS;
  int rows_per_band;
};

template <typename T, int LOAD>
__device__ __forceinline__ float load_in(const T *in0, const T *in1, long long idx) {
  float v = ldf<T>(in0 + idx);
  if (LOAD == LOAD_TANH) v = tanhf(v);
  if (LOAD == LOAD_DZ) v *= gelu_grad_f(ldf<T>(in1 + idx));
  return v;
}

size_t fwd_slab_smem(int S, int NL, int mL, int QS) {
  return sizeof(float2) * ((size_t)NL + S + (size_t)FS_NC * mL + (size_t)FS_RT * mL +
                           (size_t)QS * mL) +
         sizeof(float) * FS_RT * (FS_NC + 1);
}

template <typename T, int LOAD>
__global__ void __launch_bounds__(FS_THREADS) k_fwd_slab(FwdSlabArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int NL = a.NL, S = a.S, mL = a.mL, QS = a.QS;
  float2 *twL = reinterpret_cast<float2 *>(smem);
  float2 *twS = twL + NL;
  float2 *Tt = twS + S;                 // [FS_NC][mL] conj twiddles of the chunk
  float2 *X1 = Tt + FS_NC * mL;         // [FS_RT][mL] last-axis spectra of the tile
  float2 *acc2 = X1 + FS_RT * mL;       // [QS][mL] running slab-axis sums
  float *xs = reinterpret_cast<float *>(acc2 + QS * mL);  // [FS_RT][FS_NC+1]

  const int tid = threadIdx.x;
  const long long plane = blockIdx.x;
  const int band = blockIdx.y;
  build_twiddles(twL, NL);
  build_twiddles(twS, S);
  for (int p = tid; p < QS * mL; p += FS_THREADS) acc2[p] = make_float2(0.f, 0.f);

  const T *in0 = reinterpret_cast<const T *>(a.in0) + plane * S * NL;
  const T *in1 = LOAD == LOAD_DZ ? reinterpret_cast<const T *>(a.in1) + plane * S * NL : nullptr;
  const int tx = tid & 15, ty = tid >> 4;
  const int r_begin = band * a.rows_per_band;
  const int r_end = min(S, r_begin + a.rows_per_band);

  for (int rt0 = r_begin; rt0 < r_end; rt0 += FS_RT) {
    float2 acc[4][FS_MAXJ];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < FS_MAXJ; ++j) acc[i][j] = make_float2(0.f, 0.f);

    for (int c0 = 0; c0 < NL; c0 += FS_NC) {
      __syncthreads();
      for (int e = tid; e < FS_RT * FS_NC; e += FS_THREADS) {
        const int r = e / FS_NC, c = e - r * FS_NC;
        const int row = rt0 + r, col = c0 + c;
        float v = 0.f;
        if (row < r_end && col < NL) v = load_in<T, LOAD>(in0, in1, (long long)row * NL + col);
        xs[r * (FS_NC + 1) + c] = v;
      }
      for (int e = tid; e < FS_NC * mL; e += FS_THREADS) {
        const int c = e / mL, k = e - c * mL, col = c0 + c;
        float2 t = make_float2(0.f, 0.f);
        if (col < NL) {
          const float2 w = twL[(k * col) % NL];
          t = make_float2(w.x, -w.y);
        }
        Tt[e] = t;
      }
      __syncthreads();
      const int ncol = min(FS_NC, NL - c0);
      for (int c = 0; c < ncol; ++c) {
        float xv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[i] = xs[(ty + 16 * i) * (FS_NC + 1) + c];
#pragma unroll
        for (int j = 0; j < FS_MAXJ; ++j) {
          const int k = tx + 16 * j;
          if (k < mL) {
            const float2 t = Tt[c * mL + k];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[i][j].x = fmaf(xv[i], t.x, acc[i][j].x);
              acc[i][j].y = fmaf(xv[i], t.y, acc[i][j].y);
            }
          }
        }
      }
    }
    __syncthreads();  // previous tile's slab-axis pass is done with X1
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < FS_MAXJ; ++j) {
        const int k = tx + 16 * j;
        if (k < mL) X1[(ty + 16 * i) * mL + k] = acc[i][j];
      }
    __syncthreads();
    const int nrows = min(FS_RT, r_end - rt0);
    for (int p = tid; p < QS * mL; p += FS_THREADS) {
      const int q = p / mL, k = p - q * mL;
      const int ks = QS == 1 ? 0 : kept_k(q, a.mS, S);
      float2 s = acc2[p];
      int idx = mulmod(ks, rt0, S);
      for (int r = 0; r < nrows; ++r) {
        cfma_conj_b(s, X1[r * mL + k], twS[idx]);
        idx += ks;
        if (idx >= S) idx -= S;
      }
      acc2[p] = s;
    }
  }
  __syncthreads();
  float2 *dst = a.zpart + ((long long)band * a.planes + plane) * QS * mL;
  for (int p = tid; p < QS * mL; p += FS_THREADS) dst[p] = acc2[p];
}

// Sum the bands; for 3D grids also contract the outer axis (kept modes QO).
__global__ void __launch_bounds__(256) k_fwd_finish(const float2 *__restrict__ zpart,
                                                    float2 *__restrict__ xhat, long long BC,
                                                    int nbands, long long planes, int O, int mO,
                                                    int QO, int QSmL) {
  extern __shared__ __align__(16) unsigned char smem[];
  float2 *twO = reinterpret_cast<float2 *>(smem);
  if (QO > 1) build_twiddles(twO, O);
  __syncthreads();
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= BC * QSmL) return;
  const long long bc = t / QSmL;
  const int p = (int)(t - bc * QSmL);
  if (QO == 1) {
    float2 s = make_float2(0.f, 0.f);
    for (int band = 0; band < nbands; ++band) {
      const float2 z = zpart[((long long)band * planes + bc) * QSmL + p];
      s.x += z.x;
      s.y += z.y;
    }
    xhat[bc * QSmL + p] = s;
    return;
  }
  for (int q0 = 0; q0 < QO; q0 += 16) {
    float2 acc[16];
    int idx[16], stp[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      acc[q] = make_float2(0.f, 0.f);
      idx[q] = 0;
      stp[q] = q0 + q < QO ? kept_k(q0 + q, mO, O) : 0;
    }
    for (int n0 = 0; n0 < O; ++n0) {
      float2 z = make_float2(0.f, 0.f);
      for (int band = 0; band < nbands; ++band) {
        const float2 v = zpart[((long long)band * planes + bc * O + n0) * QSmL + p];
        z.x += v.x;
        z.y += v.y;
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        if (q0 + q < QO) cfma_conj_b(acc[q], z, twO[idx[q]]);
        idx[q] += stp[q];
        if (idx[q] >= O) idx[q] -= O;
      }
    }
#pragma unroll
    for (int q = 0; q < 16; ++q)
      if (q0 + q < QO) xhat[(bc * QO + q0 + q) * QSmL + p] = acc[q];
  }
}

// Z[b,c,n0,q,k] = sum_{q0} V[b,c,q0,q,k] exp(+2 pi i k0(q0) n0 / O)
__global__ void __launch_bounds__(256) k_inv_expand(const float2 *__restrict__ V,
                                                    float2 *__restrict__ Z, long long BC, int O,
                                                    int mO, int QO, int QSmL) {
  extern __shared__ __align__(16) unsigned char smem[];
  float2 *twO = reinterpret_cast<float2 *>(smem);
  build_twiddles(twO, O);
  __syncthreads();
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= BC * O * QSmL) return;
  const int p = (int)(t % QSmL);
  const long long rest = t / QSmL;
  const int n0 = (int)(rest % O);
  const long long bc = rest / O;
  float2 s = make_float2(0.f, 0.f);
  KeptIndex ki(mO, O, n0);
  for (int q0 = 0; q0 < QO; ++q0) cfma(s, V[(bc * QO + q0) * QSmL + p], twO[ki.next()]);
  Z[t] = s;
}

template <typename T>
cudaError_t launch_fwd_slab_t(const Launch &L, int load_mode, dim3 grid, size_t smem,
                              const FwdSlabArgs &args) {
  switch (load_mode) {
    case LOAD_PLAIN:
      cudaFuncSetAttribute(k_fwd_slab<T, LOAD_PLAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      k_fwd_slab<T, LOAD_PLAIN><<<grid, FS_THREADS, smem, L.stream>>>(args);
      break;
    case LOAD_TANH:
      cudaFuncSetAttribute(k_fwd_slab<T, LOAD_TANH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      k_fwd_slab<T, LOAD_TANH><<<grid, FS_THREADS, smem, L.stream>>>(args);
      break;
    default:
      cudaFuncSetAttribute(k_fwd_slab<T, LOAD_DZ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
      k_fwd_slab<T, LOAD_DZ><<<grid, FS_THREADS, smem, L.stream>>>(args);
      break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_slab(const Launch &L, const Geom &g, int dtype, int load_mode, long long C,
                            const void *in0, const void *in1, float2 *zpart, int nb);

int fwd_bands(const Geom &g, long long planes, int num_sms) {
  // Enough CTAs for several waves, with bands of whole row tiles.
  const int tiles = (g.S + FS_RT - 1) / FS_RT;
  long long target = 4LL * num_sms;
  int nb = 1;
  while (nb < tiles && planes * nb < target) nb *= 2;
  if (nb > tiles) nb = tiles;
  return nb;
}

size_t fwd_zpart_bytes(const Geom &g, long long C) {
  const long long planes = g.B * C * g.O;
  long long nb = fwd_bands(g, planes, 148);
  const long long ntc = s1_tc_bands(g);
  if (ntc > nb) nb = ntc;
  return sizeof(float2) * (size_t)nb * planes * g.QS * g.mL;
}

cudaError_t launch_fwd_transform(const Launch &L, const Geom &g, int dtype, int load_mode,
                                 long long C, const void *in0, const void *in1, float2 *zpart,
                                 float2 *xhat) {
  const long long planes = g.B * C * g.O;
  int nb;
  cudaError_t err;
  // Default path, chosen by the per-stage measurement of both designs on the
  // workloads' shapes: the streaming pruned FFT for 2D grids; the tensor-core
  // DFT contraction for 3D grids and wherever the streaming kernel does not
  // fit (the clustered FFT kernel is measured slower than either and is kept
  // for kernel path 4 only).
  if (L.tc == 1 && g.d == 2 && fwd_plane_supported(g, dtype, in0, in1, load_mode)) {
    return launch_fwd_plane(L, g, dtype, load_mode, C, in0, in1, xhat);
  } else if (L.tc == 4 && fwd_fft_supported(g, in0, in1, load_mode)) {
    if (g.QO == 1) return launch_fwd_fft(L, g, dtype, load_mode, C, in0, in1, xhat);
    err = launch_fwd_fft(L, g, dtype, load_mode, C, in0, in1, zpart);
    if (err != cudaSuccess) return err;
    nb = 1;
  } else if ((L.tc == 1 || L.tc == 3 || L.tc == 4) && fwd_pipe_supported(g, dtype, load_mode, in0)) {
    nb = s1_tc_bands(g);
    err = launch_fwd_pipe(L, g, dtype, load_mode, C, in0, zpart);
    if (err != cudaSuccess) return err;
  } else if (L.tc && s1_tc_supported(g, dtype)) {
    nb = s1_tc_bands(g);
    err = launch_s1_tc(L, g, dtype, load_mode, C, in0, in1, zpart, L.err);
    if (err != cudaSuccess) return err;
  } else {
    nb = fwd_bands(g, planes, 148);
    err = launch_fwd_slab(L, g, dtype, load_mode, C, in0, in1, zpart, nb);
    if (err != cudaSuccess) return err;
  }
  const long long BC = g.B * C;
  const int QSmL = g.QS * g.mL;
  const long long n = BC * QSmL;
  const size_t smem2 = g.QO > 1 ? sizeof(float2) * g.O : 0;
  launch_begin(L);
  k_fwd_finish<<<(unsigned)((n + 255) / 256), 256, smem2, L.stream>>>(zpart, xhat, BC, nb, planes,
                                                                       g.O, g.mO, g.QO, QSmL);
  launch_end(L, "fwd_finish");
  return cudaGetLastError();
}

cudaError_t launch_fwd_slab(const Launch &L, const Geom &g, int dtype, int load_mode, long long C,
                            const void *in0, const void *in1, float2 *zpart, int nb) {
  const long long planes = g.B * C * g.O;
  const int tiles = (g.S + FS_RT - 1) / FS_RT;
  const int tiles_per_band = (tiles + nb - 1) / nb;
  FwdSlabArgs args{in0, in1, zpart, planes, g.S, g.NL, g.mL, g.mS, g.QS, tiles_per_band * FS_RT};
  const size_t smem = fwd_slab_smem(g.S, g.NL, g.mL, g.QS);
  dim3 grid((unsigned)planes, (unsigned)nb);
  cudaError_t err;
  launch_begin(L);
  if (dtype == DT_F32)
    err = launch_fwd_slab_t<float>(L, load_mode, grid, smem, args);
  else if (dtype == DT_F16)
    err = launch_fwd_slab_t<__half>(L, load_mode, grid, smem, args);
  else
    err = launch_fwd_slab_t<__nv_bfloat16>(L, load_mode, grid, smem, args);
  launch_end(L, load_mode == LOAD_DZ ? "fwd_transform_dz" : "fwd_transform");
  return err;
}

size_t inv_expand_bytes(const Geom &g, long long C) {
  if (g.QO == 1) return 0;
  return sizeof(float2) * (size_t)(g.B * C * g.O * g.QS * g.mL);
}

cudaError_t launch_inv_expand(const Launch &L, const Geom &g, long long C, const float2 *V,
                              float2 *Z) {
  const long long BC = g.B * C;
  const int QSmL = g.QS * g.mL;
  const long long n = BC * g.O * QSmL;
  launch_begin(L);
  k_inv_expand<<<(unsigned)((n + 255) / 256), 256, sizeof(float2) * g.O, L.stream>>>(
      V, Z, BC, g.O, g.mO, g.QO, QSmL);
  launch_end(L, "inv_expand");
  return cudaGetLastError();
}

}  // namespace fno
