// The block's spectral middle for 2D grids in one launch: per-mode channel
// mixing (step S3) followed by the inverse transform along the slab axis (the
// first half of S4), producing U, the spectrum inverted along the slab axis,
// that the fused epilogue contracts with the last-axis basis.
//
//   yhat[b,o,q,k] = (c_k / N) sum_i xhat[b,i,q,k] R[i,o,q,k]
//   U[b,o,n,k]    = sum_q yhat[b,o,q,k] exp(+2 pi i kq(q) n / S)
//
// A CTA owns 4 samples x 4 output channels x 4 last-axis modes and every
// slab-axis mode q, so the inverse of each (b, o, k) column has all its inputs
// in shared memory.  The inverse is a pruned radix-16 FFT: with S = 16 Q and
// n = Q a + r,
//   U[Q a + r] = sum_p exp(+2 pi i p a / 16) V_r[p],
//   V_r[p]     = sum_{kq = p (mod 16)} yhat[kq] exp(+2 pi i kq r / S),
// i.e. the kept wavenumbers are folded by residue into sixteen bins (at most
// a few per bin), then one register FFT16 per (column, r) expands them to
// sixteen grid rows.
#include "fft16.cuh"
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int SM_THREADS = 256;
constexpr int SM_BG = 4, SM_OG = 4, SM_KG = 4;
constexpr int SM_NCOL = SM_BG * SM_OG * SM_KG;
constexpr int SM_MAXQS = 64;
constexpr int SM_MAXPER = 8;   // kept slab-axis modes per residue mod 16

struct MidPlan {
  size_t ys, twr, slots, total;
};

__host__ __device__ inline MidPlan mid_plan(int QS, int S) {
  MidPlan p{};
  size_t off = 0;
  p.ys = off; off += sizeof(float2) * SM_NCOL * (size_t)(QS + 1);
  p.twr = off; off += sizeof(float2) * (size_t)QS * (S / 16);
  p.slots = off; off += sizeof(int) * 16 * (SM_MAXPER + 1);
  p.total = off;
  return p;
}

template <typename T>
__global__ void __launch_bounds__(SM_THREADS)
    k_spec_mid(const float2 *__restrict__ xhat, const T *__restrict__ R, float2 *__restrict__ U,
               long long B, int Ci, int Co, int S, int mS, int QS, int mL, int NL, float inv_n) {
  extern __shared__ __align__(16) unsigned char smem[];
  const MidPlan pl = mid_plan(QS, S);
  float2 *ys = reinterpret_cast<float2 *>(smem + pl.ys);     // [col][QS + 1]
  float2 *twr = reinterpret_cast<float2 *>(smem + pl.twr);   // [slot][Qp]
  int *slot_cnt = reinterpret_cast<int *>(smem + pl.slots);  // [16]
  int *slot_tab = slot_cnt + 16;                             // [16][SM_MAXPER]
  const int tid = threadIdx.x;
  const int Qp = S / 16;
  const long long K = (long long)QS * mL;
  const int k0 = blockIdx.x * SM_KG, o0 = blockIdx.y * SM_OG;
  const long long b0 = (long long)blockIdx.z * SM_BG;
  const int QSp = QS + 1;

  // twiddles exp(+2 pi i kq(slot) r / S) and the slots of each residue
  for (int e = tid; e < QS * Qp; e += SM_THREADS) {
    const int slot = e / Qp, r = e - slot * Qp;
    const int kq = kept_k(slot, mS, S);
    double sn, cs;
    sincospi(2.0 * (double)mulmod(kq, r, S) / S, &sn, &cs);
    twr[e] = make_float2((float)cs, (float)sn);
  }
  if (tid < 16) {
    int c = 0;
    for (int slot = 0; slot < QS; ++slot)
      if ((kept_k(slot, mS, S) & 15) == tid) slot_tab[tid * SM_MAXPER + c++] = slot;
    slot_cnt[tid] = c;
  }

  // ---- mixing: task = (position (q, kk), output-channel pair)
  const int npos = QS * SM_KG;
  for (int task = tid; task < npos * (SM_OG / 2); task += SM_THREADS) {
    const int pos = task % npos, op = task / npos;
    const int q = pos / SM_KG, kk = pos - q * SM_KG, k = k0 + kk;
    const int oa = o0 + 2 * op;
    float2 acc[SM_BG][2];
#pragma unroll
    for (int bb = 0; bb < SM_BG; ++bb) acc[bb][0] = acc[bb][1] = make_float2(0.f, 0.f);
    if (k < mL) {
      const long long qk = (long long)q * mL + k;
      const bool va = oa < Co, vb = oa + 1 < Co;
#pragma unroll 4
      for (int i = 0; i < Ci; ++i) {
        const float2 ra = va ? ldc<T>(R + 2 * (((long long)i * Co + oa) * K + qk)) : make_float2(0.f, 0.f);
        const float2 rb = vb ? ldc<T>(R + 2 * (((long long)i * Co + oa + 1) * K + qk)) : make_float2(0.f, 0.f);
#pragma unroll
        for (int bb = 0; bb < SM_BG; ++bb) {
          if (b0 + bb < B) {
            const float2 xv = __ldg(xhat + ((b0 + bb) * Ci + i) * K + qk);
            cfma(acc[bb][0], xv, ra);
            cfma(acc[bb][1], xv, rb);
          }
        }
      }
    }
    const float w = k < mL ? mode_weight(k, NL, inv_n) : 0.f;
#pragma unroll
    for (int bb = 0; bb < SM_BG; ++bb)
#pragma unroll
      for (int oo = 0; oo < 2; ++oo) {
        const int col = (bb * SM_OG + 2 * op + oo) * SM_KG + kk;
        ys[col * QSp + q] = make_float2(w * acc[bb][oo].x, w * acc[bb][oo].y);
      }
  }
  __syncthreads();

  // ---- inverse along the slab axis: task = (column, r), column fastest
  for (int task = tid; task < SM_NCOL * Qp; task += SM_THREADS) {
    const int col = task % SM_NCOL, r = task / SM_NCOL;
    const int kk = col % SM_KG, bo = col / SM_KG;
    const int ol = bo % SM_OG, bb = bo / SM_OG;
    const long long b = b0 + bb;
    const int o = o0 + ol, k = k0 + kk;
    const float2 *y = ys + col * QSp;
    float2 v[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      float2 s = make_float2(0.f, 0.f);
      const int n = slot_cnt[p];
      for (int e = 0; e < n; ++e) {
        const int slot = slot_tab[p * SM_MAXPER + e];
        cfma(s, y[slot], twr[slot * Qp + r]);
      }
      v[p] = s;
    }
    fft::fft16<+1>(v);
    if (b < B && o < Co && k < mL) {
      float2 *dst = U + ((b * Co + o) * (long long)S + r) * mL + k;
#pragma unroll
      for (int a = 0; a < 16; ++a) dst[(long long)a * Qp * mL] = v[a];
    }
  }
}

}  // namespace

bool spec_mid_supported(const Geom &g) {
  if (g.d != 2 || g.QO != 1) return false;
  if (g.S % 16 != 0 || g.QS > SM_MAXQS) return false;
  // residues hold at most ceil(QS / 16) + 1 kept modes
  if ((g.QS + 15) / 16 + 1 > SM_MAXPER) return false;
  if (g.B > 65535LL * SM_BG) return false;
  return mid_plan(g.QS, g.S).total <= 200 * 1024;
}

cudaError_t launch_spec_mid(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                            const float2 *xhat, const void *R, float2 *U) {
  const MidPlan p = mid_plan(g.QS, g.S);
  dim3 grid((unsigned)((g.mL + SM_KG - 1) / SM_KG), (unsigned)((Co + SM_OG - 1) / SM_OG),
            (unsigned)((g.B + SM_BG - 1) / SM_BG));
  launch_begin(L);
  auto go = [&](auto kern, const auto *r) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)p.total);
    if (e != cudaSuccess) return e;
    kern<<<grid, SM_THREADS, p.total, L.stream>>>(xhat, r, U, g.B, Ci, Co, g.S, g.mS, g.QS, g.mL,
                                                  g.NL, g.inv_n);
    return cudaGetLastError();
  };
  cudaError_t e;
  if (dtype == DT_F32) e = go(k_spec_mid<float>, (const float *)R);
  else if (dtype == DT_F16) e = go(k_spec_mid<__half>, (const __half *)R);
  else e = go(k_spec_mid<__nv_bfloat16>, (const __nv_bfloat16 *)R);
  launch_end(L, "spec_mid");
  return e;
}

}  // namespace fno
