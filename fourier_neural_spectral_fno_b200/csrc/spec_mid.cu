// The block's spectral middle for 2D grids: per-mode channel mixing (step S3)
// and the inverse transform along the slab axis (the first half of S4), as
// two launches that each read their inputs from HBM or L2 once.
//
//   yhat[b,o,q,k] = (c_k / N) sum_i xhat[b,i,q,k] R[i,o,q,k]      (k_mix_modes)
//   U[b,o,n,k]    = sum_q yhat[b,o,q,k] exp(+2 pi i kq(q) n / S)    (k_inv_slab_fft)
//
// k_mix_modes: a CTA owns a group of consecutive modes and four samples; it
// stages their xhat and every weight of those modes in shared memory (eight
// loads in flight per thread), then forms all (b, o) products from there.
//
// k_inv_slab_fft: a CTA owns one (b, o) slab.  The inverse is a pruned
// radix-16 FFT: with S = 16 Q and n = Q a + r,
//   U[Q a + r] = sum_p exp(+2 pi i p a / 16) V_r[p],
//   V_r[p]     = sum_{kq = p (mod 16)} yhat[kq] exp(+2 pi i kq r / S),
// i.e. the kept wavenumbers (signed, in [-mS, mS)) are folded by residue into
// sixteen bins of at most four, then one register FFT16 per (r, k) expands
// them to sixteen grid rows; consecutive threads take consecutive k, so every
// row of U is written by one coalesced store.
#include "fft16.cuh"
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int MM_THREADS = 256;
constexpr int MM_BS = 4;                        // samples per CTA
constexpr size_t MM_R_STAGE = 64 * 1024;        // staged weights per CTA
constexpr int IS_THREADS = 256;
constexpr int SM_MAXQS = 64;

// modes per CTA: 4 (whole 32-byte sectors of the mode-contiguous rows) unless
// the staged weights would exceed MM_R_STAGE
int mix_modes_group(int Ci, int Co) {
  int mg = 4;
  while (mg > 1 && sizeof(float2) * (size_t)Ci * Co * mg > MM_R_STAGE) mg /= 2;
  return sizeof(float2) * (size_t)Ci * Co * mg > MM_R_STAGE ? 0 : mg;
}

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

// global load of 8 values per thread before any is stored: the staging keeps
// eight loads in flight instead of one
template <typename F>
__device__ __forceinline__ void stage8(float2 *dst, int n, F load) {
  for (int base = threadIdx.x; base < n; base += 8 * MM_THREADS) {
    float2 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = base + u * MM_THREADS;
      v[u] = e < n ? load(e) : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = base + u * MM_THREADS;
      if (e < n) dst[e] = v[u];
    }
  }
}

template <typename T, int MG>
__global__ void __launch_bounds__(MM_THREADS)
    k_mix_modes(const float2 *__restrict__ xhat, const T *__restrict__ R, float2 *__restrict__ yhat,
                float2 *__restrict__ twr, int B, int Ci, int Co, int K, int mL, int NL,
                float inv_n, int S, int mS, int QS) {
  extern __shared__ __align__(16) unsigned char smem[];
  float2 *xs = reinterpret_cast<float2 *>(smem);     // [MM_BS][Ci][MG]
  float2 *rs = xs + (size_t)MM_BS * Ci * MG;         // [Ci][Co][MG]
  const int m0 = blockIdx.x * MG, b0 = blockIdx.y * MM_BS;
  const int mg = min(MG, K - m0), nb = min(MM_BS, B - b0);
  const int tid = threadIdx.x;
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    // the slab-axis inverse's twiddles exp(+2 pi i kq(slot) r / S), [slot][S/16]
    const int Qp = S / 16;
    for (int e = tid; e < QS * Qp; e += MM_THREADS) {
      const int slot = e / Qp, r = e - slot * Qp;
      float sn, cs;
      sincospif(2.0f * (float)mulmod(kept_k(slot, mS, S), r, S) / (float)S, &sn, &cs);
      twr[e] = make_float2(cs, sn);
    }
  }
  const float2 *xsrc = xhat + (size_t)b0 * Ci * K + m0;
  stage8(xs, nb * Ci * MG, [&](int e) {
    const int row = e / MG, m = e % MG;                  // MG is a power of two
    return m < mg ? __ldg(xsrc + (size_t)row * K + m) : make_float2(0.f, 0.f);
  });
  const T *rsrc = R + 2 * (size_t)m0;
  stage8(rs, Ci * Co * MG, [&](int e) {
    const int row = e / MG, m = e % MG;
    return m < mg ? ldc<T>(rsrc + 2 * ((size_t)row * K + m)) : make_float2(0.f, 0.f);
  });
  __syncthreads();
  // output (b, o, m), m fastest: the weight reads of a warp are contiguous;
  // the (b, o) pair advances by a constant stride per thread
  const int m = tid % MG;
  const int bo_step = MM_THREADS / MG;
  const float w = m < mg ? mode_weight((m0 + m) % mL, NL, inv_n) : 0.f;
  int b = 0, o = tid / MG;
  while (o >= Co) { o -= Co; ++b; }
  const int db = bo_step / Co, dob = bo_step % Co;
  const int rstep = Co * MG;
  for (; b < nb;) {
    const float2 *xp = xs + b * Ci * MG + m;
    const float2 *rp = rs + o * MG + m;
    float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
    int i = 0;
#pragma unroll 4
    for (; i + 1 < Ci; i += 2) {
      cfma(s0, xp[i * MG], rp[i * rstep]);
      cfma(s1, xp[(i + 1) * MG], rp[(i + 1) * rstep]);
    }
    if (i < Ci) cfma(s0, xp[i * MG], rp[i * rstep]);
    if (m < mg)
      yhat[((size_t)(b0 + b) * Co + o) * K + m0 + m] =
          make_float2(w * (s0.x + s1.x), w * (s0.y + s1.y));
    b += db;
    o += dob;
    if (o >= Co) { o -= Co; ++b; }
  }
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
// so every candidate is kept and no test is needed.  twr_g: the twiddle table
// of the mixing kernel, or NULL to build it here.
template <int NDM, bool FULL>
__global__ void __launch_bounds__(IS_THREADS)
    k_inv_slab_fft(const float2 *__restrict__ yhat, const float2 *__restrict__ twr_g,
                   float2 *__restrict__ U, int S, int mS, int QS, int mL) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int Qp = S / 16;
  float2 *ys = reinterpret_cast<float2 *>(smem);      // [QS][mL]
  float2 *twr = ys + (size_t)QS * mL;                  // [slot][Qp]
  const size_t slab = blockIdx.x;
  const int tid = threadIdx.x;
  const float2 *src = yhat + slab * QS * mL;
  for (int e = tid; e < QS * mL; e += IS_THREADS) ys[e] = __ldg(src + e);
  if (twr_g) {
    for (int e = tid; e < QS * Qp; e += IS_THREADS) twr[e] = __ldg(twr_g + e);
  } else {   // no table from the mixing kernel: build it here
    for (int e = tid; e < QS * Qp; e += IS_THREADS) {
      const int slot = e / Qp, rr = e - slot * Qp;
      float sn, cs;
      sincospif(2.0f * (float)mulmod(kept_k(slot, mS, S), rr, S) / (float)S, &sn, &cs);
      twr[e] = make_float2(cs, sn);
    }
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
// and a quarter of the r's, and thread t takes channel t % 8 and mode
// (t / 8) % mL, so that the sixteen-byte rows of the core matrices of one grid
// row leave a warp as one contiguous 256-byte store (the (re, im) pairs of two
// modes of eight channels).  IMG 1: float32 images (tf32 high parts in rows
// [0, Co), low parts in [Co, 2 Co)); 2 / 3: float16 / bfloat16 images; the
// bias is folded into column 0.
constexpr int IMG_RSPLIT = 4;
template <int NDM, bool FULL, int IMG, typename TB>
__global__ void __launch_bounds__(IS_THREADS)
    k_inv_slab_img(const float2 *__restrict__ yhat, const float2 *__restrict__ twr_g,
                   unsigned char *__restrict__ img, const TB *__restrict__ bias, int S, int mS,
                   int QS, int mL, int Co) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int Qp = S / 16;
  float2 *ys = reinterpret_cast<float2 *>(smem);      // [slot][k][8 channels]
  float2 *twr = ys + (size_t)QS * mL * 8;              // [slot][Qp]
  const int groups = Co / 8;
  const int b = blockIdx.x / groups, o0 = (blockIdx.x - b * groups) * 8;
  const int tid = threadIdx.x;
  for (int e = tid; e < 8 * QS * mL; e += IS_THREADS) {
    const int oo = e / (QS * mL), sk = e - oo * (QS * mL);
    ys[sk * 8 + oo] = __ldg(yhat + ((size_t)b * Co + o0 + oo) * QS * mL + sk);
  }
  for (int e = tid; e < QS * Qp; e += IS_THREADS) twr[e] = __ldg(twr_g + e);
  __syncthreads();
  constexpr int EB = IMG == 1 ? 4 : 2;
  const uint32_t sbo = (uint32_t)(2 * mL * EB / 16) * 128u;
  const size_t row_bytes = (size_t)(IMG == 1 ? 2 * Co : Co) * 2 * mL * EB;
  const int oo = tid & 7;
  const int o = o0 + oo;
  const float bias_o = bias ? to_f<TB>(bias[o]) : 0.f;
  const int per_r = 8 * mL;
  const int r_lo = blockIdx.y * ((Qp + IMG_RSPLIT - 1) / IMG_RSPLIT);
  const int r_hi = min(Qp, r_lo + (Qp + IMG_RSPLIT - 1) / IMG_RSPLIT);
  for (int task = tid; task < (r_hi - r_lo) * per_r; task += IS_THREADS) {
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
          cfma(acc, ys[(slot * mL + k) * 8 + oo], twr[slot * Qp + r]);
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
    kern<<<slabs, IS_THREADS, smem2, L.stream>>>(Z, nullptr, U, g.S, g.mS, g.QS, g.mL);
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

bool spec_mid_img_supported(const Geom &g, int Co) {
  if (Co % 8 != 0) return false;
  const size_t smem = sizeof(float2) * ((size_t)8 * g.QS * g.mL + (size_t)g.QS * (g.S / 16));
  return smem <= 200 * 1024;
}

size_t spec_mid_table_bytes(const Geom &g) {
  return g.d == 2 ? sizeof(float2) * (size_t)g.QS * (g.S / 16) : 0;
}

bool spec_mid_supported(const Geom &g, int Ci, int Co) {
  if (g.d != 2 || g.QO != 1) return false;
  if (g.S % 16 != 0 || g.QS > SM_MAXQS) return false;
  if (g.B * (long long)g.K * kMaxWidth > (1LL << 31)) return false;
  if (mix_modes_group(Ci, Co) < 1) return false;
  if ((g.B + MM_BS - 1) / MM_BS > 65535) return false;
  const size_t inv = sizeof(float2) * ((size_t)g.QS * g.mL + (size_t)g.QS * (g.S / 16));
  return inv <= 200 * 1024;
}

cudaError_t launch_spec_mid(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                            const float2 *xhat, const void *R, float2 *yhat, float2 *twr,
                            float2 *U, unsigned char *img, const void *bias) {
  const int mg = mix_modes_group(Ci, Co);
  const size_t smem = sizeof(float2) * ((size_t)MM_BS * Ci + (size_t)Ci * Co) * mg;
  dim3 grid((unsigned)((g.K + mg - 1) / mg), (unsigned)((g.B + MM_BS - 1) / MM_BS));
  launch_begin(L);
  auto go = [&](auto kern, const auto *r) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, MM_THREADS, smem, L.stream>>>(xhat, r, yhat, twr, (int)g.B, Ci, Co, (int)g.K,
                                               g.mL, g.NL, g.inv_n, g.S, g.mS, g.QS);
    return cudaGetLastError();
  };
  auto by_mg = [&](auto k4, auto k2, auto k1, const auto *r) {
    return mg == 4 ? go(k4, r) : mg == 2 ? go(k2, r) : go(k1, r);
  };
  cudaError_t e;
  if (dtype == DT_F32)
    e = by_mg(k_mix_modes<float, 4>, k_mix_modes<float, 2>, k_mix_modes<float, 1>,
              (const float *)R);
  else if (dtype == DT_F16)
    e = by_mg(k_mix_modes<__half, 4>, k_mix_modes<__half, 2>, k_mix_modes<__half, 1>,
              (const __half *)R);
  else
    e = by_mg(k_mix_modes<__nv_bfloat16, 4>, k_mix_modes<__nv_bfloat16, 2>,
              k_mix_modes<__nv_bfloat16, 1>, (const __nv_bfloat16 *)R);
  launch_end(L, "mix_modes");
  if (e != cudaSuccess) return e;

  launch_begin(L);
  if (!img) {
    const size_t smem2 = sizeof(float2) * ((size_t)g.QS * g.mL + (size_t)g.QS * (g.S / 16));
    const unsigned slabs = (unsigned)(g.B * Co);
    auto go2 = [&](auto kern) {
      cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)smem2);
      if (e2 != cudaSuccess) return e2;
      kern<<<slabs, IS_THREADS, smem2, L.stream>>>(yhat, twr, U, g.S, g.mS, g.QS, g.mL);
      return cudaGetLastError();
    };
    if (g.mS == 16) e = go2(k_inv_slab_fft<1, true>);
    else if (g.mS == 32) e = go2(k_inv_slab_fft<2, true>);
    else if (g.mS > 16) e = go2(k_inv_slab_fft<2, false>);
    else e = go2(k_inv_slab_fft<1, false>);
  } else {
    const size_t smem3 =
        sizeof(float2) * ((size_t)8 * g.QS * g.mL + (size_t)g.QS * (g.S / 16));
    dim3 grid3((unsigned)(g.B * (Co / 8)), IMG_RSPLIT);
    auto go3 = [&](auto kern, const auto *bp) {
      cudaError_t e3 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)smem3);
      if (e3 != cudaSuccess) return e3;
      kern<<<grid3, IS_THREADS, smem3, L.stream>>>(yhat, twr, img, bp, g.S, g.mS, g.QS, g.mL, Co);
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
