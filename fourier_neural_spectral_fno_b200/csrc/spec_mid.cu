// The block's spectral middle for 2D grids: after the per-mode mixing (step
// S3, k_mix_fwd in mix.cu), the inverse transform along the slab axis (the
// first half of S4) as a pruned radix-16 FFT,
//
//   U[b,o,n,k] = sum_q yhat[b,o,q,k] exp(+2 pi i kq(q) n / S).
//
// With S = 16 Q and n = Q a + r,
//   U[Q a + r] = sum_p exp(+2 pi i p a / 16) V_r[p],
//   V_r[p]     = sum_{kq = p (mod 16)} yhat[kq] exp(+2 pi i kq r / S),
// i.e. the kept wavenumbers (signed, in [-mS, mS)) are folded by residue into
// sixteen bins of at most four, then one register FFT16 per (r, k) expands
// them to sixteen grid rows.
//
// k_inv_slab_fft writes U (one CTA per (b, o) slab, consecutive threads on
// consecutive k, so every row of U leaves as one coalesced store);
// k_inv_slab_img writes, per (sample, grid row), the spectral half of the
// pipelined epilogue's tcgen05 B operand directly in its shared-memory layout,
// so the epilogue fetches it with one bulk copy and builds nothing.
#include "fft16.cuh"
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int IS_THREADS = 256;
constexpr int SM_MAXQS = 64;
constexpr int IS_FILL = 16;     // loads in flight per thread while filling shared memory

// hi = x rounded to tf32 (nearest), lo = x - hi rounded to tf32: the
// operand split of the float32 tensor-core path
__device__ __forceinline__ void tc_split(float x, uint32_t &hi, uint32_t &lo) {
  uint32_t h, l;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
  const float rem = x - __uint_as_float(h);
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(l) : "f"(rem));
  hi = h;
  lo = l;
}

// byte offset of B-operand element (row n, column c) in a K-major no-swizzle
// image of `sbo`-byte 8-row groups (the tcgen05 core-matrix layout)
__device__ __forceinline__ uint32_t img_off(int n, int c, int eb, uint32_t sbo) {
  const int cb = c * eb;
  return (uint32_t)(n >> 3) * sbo + (uint32_t)(cb >> 4) * 128u + (uint32_t)(n & 7) * 16u +
         (uint32_t)(cb & 15);
}

// NDM: the kept wavenumbers of residue p (mod 16) are among p + 16 d,
// d in [-NDM, NDM) (NDM = 1 for mS <= 16, 2 for mS <= 32); FULL: mS = 16 NDM,
// so every candidate is kept and no test is needed.
template <int NDM, bool FULL>
__global__ void __launch_bounds__(IS_THREADS)
    k_inv_slab_fft(const float2 *__restrict__ yhat, float2 *__restrict__ U, int S, int mS,
                   int QS, int mL) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int Qp = S / 16;
  float2 *ys = reinterpret_cast<float2 *>(smem);      // [QS][mL]
  float2 *twr = ys + (size_t)QS * mL;                  // [slot][Qp]
  const size_t slab = blockIdx.x;
  const int tid = threadIdx.x;
  const float2 *src = yhat + slab * QS * mL;
  for (int e0 = tid; e0 < QS * mL; e0 += IS_FILL * IS_THREADS) {   // IS_FILL loads in flight
    float2 v[IS_FILL];
#pragma unroll
    for (int u = 0; u < IS_FILL; ++u)
      if (e0 + u * IS_THREADS < QS * mL) v[u] = __ldg(src + e0 + u * IS_THREADS);
#pragma unroll
    for (int u = 0; u < IS_FILL; ++u)
      if (e0 + u * IS_THREADS < QS * mL) ys[e0 + u * IS_THREADS] = v[u];
  }
  for (int e = tid; e < QS * Qp; e += IS_THREADS) {   // exp(+2 pi i kq(slot) r / S)
    const int slot = e / Qp, rr = e - slot * Qp;
    float sn, cs;
    sincospif(2.0f * (float)mulmod(kept_k(slot, mS, S), rr, S) / (float)S, &sn, &cs);
    twr[e] = make_float2(cs, sn);
  }
  __syncthreads();
  float2 *dst = U + slab * (size_t)S * mL;
  int k = tid % mL, r = tid / mL;                        // task = r mL + k
  const int dr = IS_THREADS / mL, dk = IS_THREADS % mL;
  for (; r < Qp;) {
    float2 v[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int d = -NDM; d < NDM; ++d) {
        const int kq = p + 16 * d;            // signed wavenumber
        if (FULL || (kq >= -mS && kq < mS)) {
          const int slot = kq >= 0 ? kq : kq + QS;
          cfma(acc, ys[slot * mL + k], twr[slot * Qp + r]);
        }
      }
      v[p] = acc;
    }
    fft::fft16<+1>(v);
    float2 *d = dst + (size_t)r * mL + k;
#pragma unroll
    for (int a = 0; a < 16; ++a) d[(size_t)a * Qp * mL] = v[a];
    r += dr;
    k += dk;
    if (k >= mL) { k -= mL; ++r; }
  }
}

// The same inverse writing the epilogue's B images: a CTA owns eight
// consecutive output channels (one 8-row group of the operand's core matrices)
// and a range of the r's, and thread t takes channel t % 8 and mode
// (t / 8) % mL, so that the sixteen-byte rows of the core matrices of one grid
// row leave a warp as one contiguous 256-byte store (the (re, im) pairs of two
// modes of eight channels); the grid's y dimension splits the r's.  IMG 1:
// float32 images (tf32 high parts in rows [0, Co), low parts in [Co, 2 Co));
// 2 / 3: float16 / bfloat16 images; the bias is folded into column 0.
constexpr int IMG_RSPLIT = 4;   // r ranges per (sample, channel group)
template <int NDM, bool FULL, int IMG, typename TB>
__global__ void __launch_bounds__(IS_THREADS)
    k_inv_slab_img(const float2 *__restrict__ yhat, unsigned char *__restrict__ img, const TB *__restrict__ bias, int S, int mS,
                   int QS, int mL, int Co) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int Qp = S / 16;
  const int nsk = QS * mL, ysl = nsk + 4;                // padded channel rows
  float2 *ys = reinterpret_cast<float2 *>(smem);      // [8 channels][slot][k]
  float2 *twr = ys + (size_t)8 * ysl;                  // [slot][Qp]
  const int groups = Co / 8;
  const int b = blockIdx.x / groups, o0 = (blockIdx.x - b * groups) * 8;
  const int tid = threadIdx.x;
  // sixteen loads in flight per thread before their stores; consecutive
  // threads take consecutive (slot, k), so the stores meet no bank conflict
  const float2 *src = yhat + ((size_t)b * Co + o0) * nsk;
  for (int s0 = tid; s0 < nsk; s0 += 2 * IS_THREADS) {
    float2 v[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (s0 + h * IS_THREADS < nsk) v[h][c] = __ldg(src + (size_t)c * nsk + s0 + h * IS_THREADS);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (s0 + h * IS_THREADS < nsk) ys[c * ysl + s0 + h * IS_THREADS] = v[h][c];
  }
  const int rchunk = (Qp + (int)gridDim.y - 1) / (int)gridDim.y;
  const int r_lo = blockIdx.y * rchunk;
  const int r_hi = min(Qp, r_lo + rchunk);
  const int rn = r_hi - r_lo;
  for (int e = tid; e < QS * rn; e += IS_THREADS) {   // this CTA's r only
    const int slot = e / rn, rr = r_lo + (e - slot * rn);
    float sn, cs;
    sincospif(2.0f * (float)mulmod(kept_k(slot, mS, S), rr, S) / (float)S, &sn, &cs);
    twr[slot * Qp + rr] = make_float2(cs, sn);
  }
  __syncthreads();
  constexpr int EB = IMG == 1 ? 4 : 2;
  const uint32_t sbo = (uint32_t)(2 * mL * EB / 16) * 128u;
  const size_t row_bytes = (size_t)(IMG == 1 ? 2 * Co : Co) * 2 * mL * EB;
  const int oo = tid & 7;
  const int o = o0 + oo;
  const float bias_o = bias ? to_f<TB>(bias[o]) : 0.f;
  const int per_r = 8 * mL;
  for (int task = tid; task < rn * per_r; task += IS_THREADS) {
    const int r = r_lo + task / per_r, k = (task / 8) % mL;
    float2 v[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int d = -NDM; d < NDM; ++d) {
        const int kq = p + 16 * d;
        if (FULL || (kq >= -mS && kq < mS)) {
          const int slot = kq >= 0 ? kq : kq + QS;
          cfma(acc, ys[oo * ysl + slot * mL + k], twr[slot * Qp + r]);
        }
      }
      v[p] = acc;
    }
    fft::fft16<+1>(v);
    const uint32_t hi = img_off(o, 2 * k, EB, sbo);
    const uint32_t lo = IMG == 1 ? img_off(Co + o, 2 * k, EB, sbo) : 0u;
    unsigned char *base = img + ((size_t)b * S + r) * row_bytes;
#pragma unroll
    for (int a = 0; a < 16; ++a) {
      float2 u = v[a];
      if (k == 0) u.x += bias_o;
      unsigned char *row = base + (size_t)a * Qp * row_bytes;
      if (IMG == 1) {
        uint32_t hx, lx, hy, ly;
        tc_split(u.x, hx, lx);
        tc_split(u.y, hy, ly);
        *reinterpret_cast<uint2 *>(row + hi) = make_uint2(hx, hy);
        *reinterpret_cast<uint2 *>(row + lo) = make_uint2(lx, ly);
      } else if (IMG == 2) {
        *reinterpret_cast<__half2 *>(row + hi) = __floats2half2_rn(u.x, u.y);
      } else {
        *reinterpret_cast<__nv_bfloat162 *>(row + hi) = __floats2bfloat162_rn(u.x, u.y);
      }
    }
  }
}

}  // namespace

bool inv_slab_fft_supported(const Geom &g) {
  if (g.d != 2 || g.QO != 1 || g.S % 16 != 0 || g.QS > SM_MAXQS) return false;
  const size_t inv = sizeof(float2) * ((size_t)g.QS * g.mL + (size_t)g.QS * (g.S / 16));
  return inv <= 200 * 1024;
}

cudaError_t launch_inv_slab_fft(const Launch &L, const Geom &g, long long C, const float2 *Z,
                                float2 *U) {
  const size_t smem2 = sizeof(float2) * ((size_t)g.QS * g.mL + (size_t)g.QS * (g.S / 16));
  const unsigned slabs = (unsigned)(g.B * C);
  launch_begin(L);
  auto go2 = [&](auto kern) {
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem2);
    if (e2 != cudaSuccess) return e2;
    kern<<<slabs, IS_THREADS, smem2, L.stream>>>(Z, U, g.S, g.mS, g.QS, g.mL);
    return cudaGetLastError();
  };
  cudaError_t e;
  if (g.mS == 16) e = go2(k_inv_slab_fft<1, true>);
  else if (g.mS == 32) e = go2(k_inv_slab_fft<2, true>);
  else if (g.mS > 16) e = go2(k_inv_slab_fft<2, false>);
  else e = go2(k_inv_slab_fft<1, false>);
  launch_end(L, "inv_slab_fft");
  return e;
}

// shared memory of k_inv_slab_img: eight padded channel rows of the slab
// spectrum, then the twiddle table
inline size_t img_smem(const Geom &g) {
  return sizeof(float2) * ((size_t)8 * (g.QS * g.mL + 4) + (size_t)g.QS * (g.S / 16));
}

bool spec_mid_img_supported(const Geom &g, int Co) {
  if (Co % 8 != 0) return false;
  return img_smem(g) <= 200 * 1024;
}

bool spec_mid_supported(const Geom &g, int Ci, int Co) {
  if (g.d != 2 || g.QO != 1) return false;
  if (g.S % 16 != 0 || g.QS > SM_MAXQS) return false;
  if (g.B * (long long)g.K * kMaxWidth > (1LL << 31)) return false;
  (void)Ci;
  (void)Co;
  const size_t inv = sizeof(float2) * ((size_t)g.QS * g.mL + (size_t)g.QS * (g.S / 16));
  return inv <= 200 * 1024;
}

cudaError_t launch_spec_mid(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                            const float2 *xhat, const void *R, float2 *yhat, float2 *U,
                            unsigned char *img, const void *bias) {
  cudaError_t e = launch_mix_fwd(L, g, dtype, Ci, Co, xhat, R, yhat);
  if (e != cudaSuccess) return e;
  launch_begin(L);
  if (!img) {
    const size_t smem2 = sizeof(float2) * ((size_t)g.QS * g.mL + (size_t)g.QS * (g.S / 16));
    const unsigned slabs = (unsigned)(g.B * Co);
    auto go2 = [&](auto kern) {
      cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)smem2);
      if (e2 != cudaSuccess) return e2;
      kern<<<slabs, IS_THREADS, smem2, L.stream>>>(yhat, U, g.S, g.mS, g.QS, g.mL);
      return cudaGetLastError();
    };
    if (g.mS == 16) e = go2(k_inv_slab_fft<1, true>);
    else if (g.mS == 32) e = go2(k_inv_slab_fft<2, true>);
    else if (g.mS > 16) e = go2(k_inv_slab_fft<2, false>);
    else e = go2(k_inv_slab_fft<1, false>);
  } else {
    const size_t smem3 = img_smem(g);
    dim3 grid3((unsigned)(g.B * (Co / 8)), (unsigned)(g.S / 16 < IMG_RSPLIT ? g.S / 16 : IMG_RSPLIT));
    auto go3 = [&](auto kern, const auto *bp) {
      cudaError_t e3 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)smem3);
      if (e3 != cudaSuccess) return e3;
      kern<<<grid3, IS_THREADS, smem3, L.stream>>>(yhat, img, bp, g.S, g.mS, g.QS, g.mL, Co);
      return cudaGetLastError();
    };
    auto by_out = [&](auto k1, auto k2, auto k3) {
      if (dtype == DT_F32) return go3(k1, (const float *)bias);
      if (dtype == DT_F16) return go3(k2, (const __half *)bias);
      return go3(k3, (const __nv_bfloat16 *)bias);
    };
#define FNO_INV_IMG(NDM, FULL)                                                      \
  by_out(k_inv_slab_img<NDM, FULL, 1, float>, k_inv_slab_img<NDM, FULL, 2, __half>, \
         k_inv_slab_img<NDM, FULL, 3, __nv_bfloat16>)
    if (g.mS == 16) e = FNO_INV_IMG(1, true);
    else if (g.mS == 32) e = FNO_INV_IMG(2, true);
    else if (g.mS > 16) e = FNO_INV_IMG(2, false);
    else e = FNO_INV_IMG(1, false);
#undef FNO_INV_IMG
  }
  launch_end(L, img ? "inv_slab_img" : "inv_slab_fft");
  return e;
}

}  // namespace fno
