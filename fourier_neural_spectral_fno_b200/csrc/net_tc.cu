// Projection u = Q2 GELU(Q1 v + q1) + q2 (step S5) on the sm_100a tensor cores.
//
// A tile is 128 consecutive grid points of one sample (thread t <-> point t
// <-> TMEM lane t).  The hidden layer h[p, :] = v[p, :] Q1^T is one MMA chain
// with A = v in tensor memory and B = Q1 (K-major, shared memory, built once
// per CTA); the hidden activations never leave the SM: the epilogue reads h
// back from tensor memory, adds q1, applies GELU and contracts with Q2 on the
// CUDA cores.  Float32 storage: three tf32 passes (hi/lo split); 16-bit
// storage: one kind::f16 pass, float32 accumulation.
#include "fno_common.cuh"
#include "fno_kernels.cuh"
#include "tc_util.cuh"

namespace fno {

namespace {

constexpr int TC_THREADS = 128;
constexpr int TMEM_COLS = 256;
constexpr int kMaxOut = 4;

template <typename T> struct PKind {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int KSTEP = 16;
  static constexpr int fmt = tc::FMT_F16;
};
template <> struct PKind<float> {
  static constexpr bool tf32 = true;
  static constexpr int EB = 4;
  static constexpr int KSTEP = 8;
  static constexpr int fmt = tc::FMT_TF32;
};
template <> struct PKind<__nv_bfloat16> {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int KSTEP = 16;
  static constexpr int fmt = tc::FMT_BF16;
};

__host__ __device__ inline int rup(int v, int m) { return (v + m - 1) / m * m; }
__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~(size_t)15; }

struct ProjTcGeom {
  int Cp, HP, acol, total_cols;
  uint32_t sbo;
  size_t bhi, blo, q1, q2, mbar, tbase, total;
};

__host__ __device__ inline ProjTcGeom proj_tc_geom(int width, int hidden, int out_ch, bool tf32) {
  ProjTcGeom e;
  const int eb = tf32 ? 4 : 2;
  e.Cp = rup(width, 16);
  e.HP = rup(hidden, 16);
  e.acol = e.HP;                                   // D occupies [0, HP)
  e.total_cols = e.HP + (tf32 ? 2 * e.Cp : e.Cp / 2);
  e.sbo = (uint32_t)(e.Cp * eb / 16) * 128u;
  size_t off = 0;
  const size_t bbytes = (size_t)e.HP * e.Cp * eb;
  e.bhi = off; off = al16(off + bbytes);
  e.blo = off; if (tf32) off = al16(off + bbytes);
  e.q1 = off; off = al16(off + sizeof(float) * e.HP);
  e.q2 = off; off = al16(off + sizeof(float) * (size_t)kMaxOut * e.HP);
  e.mbar = off; off = al16(off + sizeof(uint64_t));
  e.tbase = off; off = al16(off + sizeof(uint32_t));
  e.total = off < 80 * 1024 ? 80 * 1024 : off;
  return e;
}

__device__ __forceinline__ uint32_t boff(int n, int k, int eb, uint32_t sbo) {
  const int kb = k * eb;
  return (uint32_t)(n >> 3) * sbo + (kb >> 4) * 128 + (n & 7) * 16 + (kb & 15);
}

template <typename T, int CX>
__global__ void __launch_bounds__(TC_THREADS)
    k_proj_tc(const T *__restrict__ v, const T *__restrict__ Q1, const T *__restrict__ q1,
              const T *__restrict__ Q2, const T *__restrict__ q2, T *__restrict__ u, long long B,
              long long N, int width, int hidden, int out_ch, int *err) {
  using K = PKind<T>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const ProjTcGeom e = proj_tc_geom(width, hidden, out_ch, K::tf32);
  unsigned char *bhi = smem + e.bhi;
  unsigned char *blo = smem + e.blo;
  float *q1s = reinterpret_cast<float *>(smem + e.q1);
  float *q2s = reinterpret_cast<float *>(smem + e.q2);
  uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + e.mbar);
  uint32_t *tbase_s = reinterpret_cast<uint32_t *>(smem + e.tbase);
  const int t = threadIdx.x, warp = t >> 5;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (t == 0) tc::mbar_init(mbar, 1);
  // B = Q1 [hidden][width] (zero padded to HP x Cp), q1, Q2
  for (int i = t; i < e.HP * e.Cp; i += TC_THREADS) {
    const int h = i / e.Cp, c = i - h * e.Cp;
    const float val = (h < hidden && c < width) ? to_f<T>(Q1[h * width + c]) : 0.f;
    const uint32_t o = boff(h, c, K::EB, e.sbo);
    if (K::tf32) {
      uint32_t hi, lo;
      tc::split_tf32(val, hi, lo);
      *reinterpret_cast<uint32_t *>(bhi + o) = hi;
      *reinterpret_cast<uint32_t *>(blo + o) = lo;
    } else {
      *reinterpret_cast<T *>(bhi + o) = from_f<T>(val);
    }
  }
  for (int h = t; h < e.HP; h += TC_THREADS) q1s[h] = h < hidden ? to_f<T>(q1[h]) : 0.f;
  for (int i = t; i < kMaxOut * e.HP; i += TC_THREADS) {
    const int o = i / e.HP, h = i - o * e.HP;
    q2s[i] = (o < out_ch && h < hidden) ? to_f<T>(Q2[o * hidden + h]) : 0.f;
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;
  const uint32_t arow = tbase + ((uint32_t)(warp * 32) << 16);
  const uint32_t idesc = tc::instr_desc(K::fmt, 128, e.HP);
  const uint64_t bh0 = tc::smem_desc_kmajor(tc::smem_u32(bhi), 128, e.sbo);
  const uint64_t bl0 = tc::smem_desc_kmajor(tc::smem_u32(blo), 128, e.sbo);
  float q2b[kMaxOut];
#pragma unroll
  for (int o = 0; o < kMaxOut; ++o) q2b[o] = o < out_ch ? to_f<T>(q2[o]) : 0.f;

  const long long tpb = N / TC_THREADS;            // tiles per sample
  const long long ntiles = B * tpb;
  const long long per_cta = (ntiles + gridDim.x - 1) / gridDim.x;
  const long long t_begin = blockIdx.x * per_cta;
  const long long t_end = t_begin + per_cta < ntiles ? t_begin + per_cta : ntiles;

  float vr[CX];
  auto fetch = [&](long long tile) {
    const long long b = tile / tpb;
    const T *vp = v + b * width * N + (tile - b * tpb) * TC_THREADS + t;
#pragma unroll
    for (int c = 0; c < CX; ++c) vr[c] = c < width ? ldf<T>(vp + (long long)c * N) : 0.f;
  };
  uint32_t phase = 0;
  bool ok = true;
  if (t_begin < t_end) fetch(t_begin);
  for (long long tile = t_begin; tile < t_end; ++tile) {
    // A = v (this thread's point)
#pragma unroll
    for (int c0 = 0; c0 < CX; c0 += 16) {
      if (c0 < e.Cp) {
        if (K::tf32) {
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) tc::split_tf32(vr[c0 + i], hi[i], lo[i]);
          tc::tmem_st16(arow + e.acol + c0, hi);
          tc::tmem_st16(arow + e.acol + e.Cp + c0, lo);
        } else {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = K::fmt == tc::FMT_BF16 ? tc::pack_bf16(vr[c0 + 2 * i], vr[c0 + 2 * i + 1])
                                           : tc::pack_f16(vr[c0 + 2 * i], vr[c0 + 2 * i + 1]);
          tc::tmem_st8(arow + e.acol + c0 / 2, pk);
        }
      }
    }
    tc::tmem_wait_st();
    tc::fence_before_sync();
    __syncthreads();
    if ((t >> 5) == 0 && tc::elect_one()) {   // one elected thread of warp 0
      tc::fence_after_sync();
      const int ns = e.Cp / K::KSTEP;
      uint64_t bh = bh0, bl = bl0;      // +256 bytes (16 units) per K step
      uint32_t a0 = tbase + e.acol;
#pragma unroll 4
      for (int s = 0; s < ns; ++s) {
        if (K::tf32) {
          tc::mma_tf32_ts(tbase, a0, bh, idesc, s > 0 ? 1u : 0u);
          tc::mma_tf32_ts(tbase, a0, bl, idesc, 1u);
          tc::mma_tf32_ts(tbase, a0 + e.Cp, bh, idesc, 1u);
        } else {
          tc::mma_f16_ts(tbase, a0, bh, idesc, s > 0 ? 1u : 0u);
        }
        bh += 16;
        bl += 16;
        a0 += 8;
      }
      tc::mma_commit(mbar);
    }
    const long long cur = tile;
    if (tile + 1 < t_end) fetch(tile + 1);
    ok = tc::mbar_wait(mbar, phase & 1, err);
    phase++;
    tc::fence_after_sync();
    float acc[kMaxOut];
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o) acc[o] = q2b[o];
    for (int h0 = 0; h0 < e.HP; h0 += 16) {
      uint32_t dv[16];
      tc::tmem_ld16(arow + h0, dv);
      tc::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        float z0 = __uint_as_float(dv[i]) + q1s[h0 + i];
        float z1 = __uint_as_float(dv[i + 1]) + q1s[h0 + i + 1];
        gelu2(z0, z1);
#pragma unroll
        for (int o = 0; o < kMaxOut; ++o)
          if (o < out_ch)
            acc[o] = fmaf(q2s[o * e.HP + h0 + i + 1], z1, fmaf(q2s[o * e.HP + h0 + i], z0, acc[o]));
      }
    }
    const long long b = cur / tpb;
    T *up = u + b * out_ch * N + (cur - b * tpb) * TC_THREADS + t;
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o)
      if (o < out_ch) up[(long long)o * N] = from_f<T>(acc[o]);
    tc::fence_before_sync();
    if (__syncthreads_or(!ok)) break;
  }
  if (!ok) tc::mbar_wait(mbar, phase & 1, nullptr);
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, TMEM_COLS);
}

template <typename T, int CX>
cudaError_t proj_tc_t(const Launch &L, const Geom &g, int width, int hidden, int out_ch,
                      const void *v, const void *Q1, const void *q1, const void *Q2,
                      const void *q2, void *u) {
  const ProjTcGeom e = proj_tc_geom(width, hidden, out_ch, PKind<T>::tf32);
  const long long ntiles = g.B * (g.N / TC_THREADS);
  const long long cap = 2LL * L.num_sms;
  const int grid = (int)(ntiles < cap ? ntiles : cap);
  auto kern = k_proj_tc<T, CX>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)e.total);
  kern<<<grid, TC_THREADS, e.total, L.stream>>>((const T *)v, (const T *)Q1, (const T *)q1,
                                                (const T *)Q2, (const T *)q2, (T *)u, g.B, g.N,
                                                width, hidden, out_ch, L.err);
  return cudaGetLastError();
}

template <typename T>
cudaError_t proj_tc_c(const Launch &L, const Geom &g, int width, int hidden, int out_ch,
                      const void *v, const void *Q1, const void *q1, const void *Q2,
                      const void *q2, void *u) {
  if (width <= 16) return proj_tc_t<T, 16>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
  if (width <= 32) return proj_tc_t<T, 32>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
  return proj_tc_t<T, 64>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
}

}  // namespace

bool proj_tc_supported(const Geom &g, int dtype, int width, int hidden, int out_ch) {
  if (g.N % TC_THREADS != 0) return false;
  if (out_ch > kMaxOut) return false;
  const ProjTcGeom e = proj_tc_geom(width, hidden, out_ch, dtype == DT_F32);
  if (e.HP > 256 || e.total_cols > TMEM_COLS) return false;
  return e.total <= 227 * 1024;
}

cudaError_t launch_proj_fwd_tc(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                               int out_ch, const void *v, const void *Q1, const void *q1,
                               const void *Q2, const void *q2, void *u) {
  launch_begin(L);
  cudaError_t err =
      dtype == DT_F32   ? proj_tc_c<float>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u)
      : dtype == DT_F16 ? proj_tc_c<__half>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u)
                        : proj_tc_c<__nv_bfloat16>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
  launch_end(L, "proj_fwd_tc");
  return err;
}

}  // namespace fno
