// Inverse transform and fused block epilogue (step S4) on the sm_100a tensor
// cores.
//
// For a tile of 128 consecutive grid points of one (sample, outer index) slab
// the block output is one small GEMM per point:
//     pre[p, o] = sum_j basis[p, j] U[o, j] + sum_i x[p, i] W[o, i] + b[o]
// where basis = (cos, -sin)(2 pi k n / N_L) of the point's last-axis index n
// and U = the spectrum already inverted along the slab axis for the tile's
// row (k_inv_slab below).  A = [basis | x] lives in tensor memory (thread t
// <-> point t <-> TMEM lane t), B = [U | W] in shared memory, D = pre in
// tensor memory; the epilogue adds the bias, applies GELU and stores y (and
// pre), each store coalesced across the warp.  Float32 storage uses three tf32
// passes (A_hi B_hi + A_hi B_lo + A_lo B_hi); 16-bit storage one kind::f16
// pass with float32 accumulation.
#include "fno_common.cuh"
#include "fno_kernels.cuh"
#include "tc_util.cuh"

namespace fno {

namespace {

constexpr int TC_THREADS = 128;
constexpr int TMEM_COLS = 256;

template <typename T> struct EKind {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int KSTEP = 16;
  static constexpr int fmt = tc::FMT_F16;
};
template <> struct EKind<float> {
  static constexpr bool tf32 = true;
  static constexpr int EB = 4;
  static constexpr int KSTEP = 8;
  static constexpr int fmt = tc::FMT_TF32;
};
template <> struct EKind<__nv_bfloat16> {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int KSTEP = 16;
  static constexpr int fmt = tc::FMT_BF16;
};

__host__ __device__ inline int rup(int v, int m) { return (v + m - 1) / m * m; }
__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~(size_t)15; }

struct EpiTcGeom {
  int Rt;       // slab rows per tile
  int KS;       // spectral K (Rt * 2 mL), padded to KSp
  int KSp, KXp, KA, NP;
  int dcol;     // TMEM column of D
  size_t bhi, blo, twL, bias, mbar, tbase, total;
  uint32_t sbo;
};

__host__ __device__ inline EpiTcGeom epi_tc_geom(const Geom &g, int mode, int Ci, int Co, int eb,
                                                 bool tf32) {
  EpiTcGeom e;
  const int kstep = tf32 ? 8 : 16;
  e.Rt = g.NL >= 128 ? 1 : 128 / g.NL;
  e.KS = e.Rt * 2 * g.mL;
  (void)kstep;
  e.KSp = rup(e.KS, 16);                          // 16-element staging granule
  e.KXp = mode == EPI_BLOCK_FWD ? rup(Ci, 16) : 0;
  e.KA = e.KSp + e.KXp;
  const int cout = (mode == EPI_SPEC_BWD) ? Ci : Co;
  e.NP = rup(cout, 16);
  const int acols = tf32 ? 2 * e.KA : e.KA / 2;
  e.dcol = rup(acols, 32);
  e.sbo = (uint32_t)(e.KA * eb / 16) * 128u;
  size_t off = 0;
  const size_t bbytes = (size_t)e.NP * e.KA * eb;
  e.bhi = off; off = al16(off + bbytes);
  e.blo = off; if (tf32) off = al16(off + bbytes);
  e.twL = off; off = al16(off + sizeof(float2) * g.NL);
  e.bias = off; off = al16(off + sizeof(float) * 64);
  e.mbar = off; off = al16(off + sizeof(uint64_t));
  e.tbase = off; off = al16(off + sizeof(uint32_t));
  e.total = off < 80 * 1024 ? 80 * 1024 : off;   // at most two CTAs per SM (TMEM)
  return e;
}

// byte offset of element (n, k) in a K-major no-swizzle B operand
__device__ __forceinline__ size_t boff(int n, int k, int eb, uint32_t sbo) {
  const int kb = k * eb;
  return (size_t)(n >> 3) * sbo + (kb >> 4) * 128 + (n & 7) * 16 + (kb & 15);
}

template <typename T>
__device__ __forceinline__ void bstore(unsigned char *bhi, unsigned char *blo, int n, int k,
                                       uint32_t sbo, float v) {
  const size_t o = boff(n, k, EKind<T>::EB, sbo);
  if (EKind<T>::tf32) {
    uint32_t hi, lo;
    tc::split_tf32(v, hi, lo);
    *reinterpret_cast<uint32_t *>(bhi + o) = hi;
    *reinterpret_cast<uint32_t *>(blo + o) = lo;
  } else {
    *reinterpret_cast<T *>(bhi + o) = from_f<T>(v);
  }
}

struct EpiTcArgs {
  const float2 *U;  // [B][Cs][O][S][mL]
  const void *x, *W, *bias;
  void *out, *pre_out;
  int *err;
  int Ci, Co, act, tanh_pre;
};

// stage 16 A columns [c0, c0 + 16) of this thread's row into TMEM
template <typename T>
__device__ __forceinline__ void stage16(uint32_t taddr_hi, uint32_t taddr_lo, const float (&v)[16]) {
  if (EKind<T>::tf32) {
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) tc::split_tf32(v[i], hi[i], lo[i]);
    tc::tmem_st16(taddr_hi, hi);
    tc::tmem_st16(taddr_lo, lo);
  } else {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      pk[i] = EKind<T>::fmt == tc::FMT_BF16 ? tc::pack_bf16(v[2 * i], v[2 * i + 1])
                                             : tc::pack_f16(v[2 * i], v[2 * i + 1]);
    tc::tmem_st8(taddr_hi, pk);
  }
}

template <typename T, int MODE, int CX>
__global__ void __launch_bounds__(TC_THREADS) k_epi_tc(EpiTcArgs a, Geom g) {
  using K = EKind<T>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int Ci = a.Ci, Co = a.Co;
  const EpiTcGeom e = epi_tc_geom(g, MODE, Ci, Co, K::EB, K::tf32);
  unsigned char *bhi = smem + e.bhi;
  unsigned char *blo = smem + e.blo;
  float2 *twL = reinterpret_cast<float2 *>(smem + e.twL);
  float *bias_s = reinterpret_cast<float *>(smem + e.bias);
  uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + e.mbar);
  uint32_t *tbase_s = reinterpret_cast<uint32_t *>(smem + e.tbase);
  const int t = threadIdx.x, warp = t >> 5;
  const int NL = g.NL, S = g.S, mL = g.mL, O = g.O;
  const int Cs = MODE == EPI_SPEC_BWD ? Ci : Co;     // spectral output channels
  const long long SN = (long long)S * NL;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (t == 0) tc::mbar_init(mbar, 1);
  build_twiddles(twL, NL);
  // constant part of B: zero everything, then W in columns [KSp, KSp + Ci)
  {
    const size_t bbytes = (size_t)e.NP * e.KA * K::EB;
    for (size_t i = t * 16; i < bbytes; i += TC_THREADS * 16) {
      *reinterpret_cast<uint4 *>(bhi + i) = make_uint4(0, 0, 0, 0);
      if (K::tf32) *reinterpret_cast<uint4 *>(blo + i) = make_uint4(0, 0, 0, 0);
    }
  }
  __syncthreads();
  if (MODE == EPI_BLOCK_FWD) {
    const T *W = reinterpret_cast<const T *>(a.W);
    for (int i = t; i < Co * Ci; i += TC_THREADS)
      bstore<T>(bhi, blo, i / Ci, e.KSp + i % Ci, e.sbo, to_f<T>(W[i]));
    const T *bias = reinterpret_cast<const T *>(a.bias);
    for (int o = t; o < Co; o += TC_THREADS) bias_s[o] = bias ? to_f<T>(bias[o]) : 0.f;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t idesc = tc::instr_desc(K::fmt, 128, e.NP);
  const uint32_t bhi_a = tc::smem_u32(bhi), blo_a = tc::smem_u32(blo);
  const uint32_t acol_lo = K::tf32 ? (uint32_t)e.KA : 0u;   // A_lo column offset
  const T *x = reinterpret_cast<const T *>(a.x);
  T *out = reinterpret_cast<T *>(a.out);
  T *pre_out = reinterpret_cast<T *>(a.pre_out);

  const int tps = (int)(SN / TC_THREADS);          // tiles per slab
  const long long ntiles = g.B * O * tps;
  uint32_t phase = 0;
  bool ok = true;

  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const long long slab = tile / tps;
    const long long pbase = (tile - slab * tps) * (long long)TC_THREADS;
    const long long b = slab / O;
    const int outer = (int)(slab - b * O);
    const int row0 = (int)(pbase / NL);
    const long long p = pbase + t;
    const int n = (int)(p % NL);
    const int rl = (int)(p / NL) - row0;

    // (1) spectral part of B for this tile's rows: B[o][rl*2mL + 2k (+1)] = U
    for (int i = t; i < e.Rt * Cs * mL; i += TC_THREADS) {
      const int k = i % mL;
      const int rest = i / mL;
      const int o = rest % Cs, r = rest / Cs;
      const float2 u = __ldg(a.U + ((((b * Cs + o) * O + outer) * S) + row0 + r) * (long long)mL + k);
      const int col = r * 2 * mL + 2 * k;
      bstore<T>(bhi, blo, o, col, e.sbo, u.x);
      bstore<T>(bhi, blo, o, col + 1, e.sbo, u.y);
    }
    // (2) A = [basis | x] for this thread's point
    {
      const uint32_t arow = tbase + lane_off;
      for (int c0 = 0; c0 < e.KSp; c0 += 16) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int j = c0 + i;
          float val = 0.f;
          if (j < e.KS) {
            const int r = j / (2 * mL), jj = j - r * 2 * mL;
            if (r == rl) {
              const float2 w = twL[((jj >> 1) * n) % NL];
              val = (jj & 1) ? -w.y : w.x;
            }
          }
          v[i] = val;
        }
        stage16<T>(arow + (K::tf32 ? c0 : c0 / 2), arow + acol_lo + c0, v);
      }
      if (MODE == EPI_BLOCK_FWD) {
        const long long xb = (b * Ci * O + outer) * SN + p;
        for (int c0 = 0; c0 < e.KXp; c0 += 16) {
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int ci = c0 + i;
            v[i] = (ci < Ci) ? ldf<T>(x + xb + (long long)ci * O * SN) : 0.f;
          }
          const int col = e.KSp + c0;
          stage16<T>(arow + (K::tf32 ? col : col / 2), arow + acol_lo + col, v);
        }
      }
    }
    tc::tmem_wait_st();
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    // (3) one thread issues the MMAs
    if (t == 0) {
      tc::fence_after_sync();
      const int nsteps = e.KA / K::KSTEP;
      for (int s = 0; s < nsteps; ++s) {
        const uint64_t bh = tc::smem_desc_kmajor(bhi_a + s * 256, 128, e.sbo);
        const uint32_t acolh = tbase + s * 8;   // 8 columns per K step (tf32 or packed 16-bit)
        if (K::tf32) {
          const uint64_t bl = tc::smem_desc_kmajor(blo_a + s * 256, 128, e.sbo);
          tc::mma_tf32_ts(tbase + e.dcol, acolh, bh, idesc, s > 0 ? 1u : 0u);
          tc::mma_tf32_ts(tbase + e.dcol, acolh, bl, idesc, 1u);
          tc::mma_tf32_ts(tbase + e.dcol, acolh + acol_lo, bh, idesc, 1u);
        } else {
          tc::mma_f16_ts(tbase + e.dcol, acolh, bh, idesc, s > 0 ? 1u : 0u);
        }
      }
      tc::mma_commit(mbar);
    }
    // (4) epilogue
    ok = tc::mbar_wait(mbar, phase & 1, a.err);
    phase++;
    tc::fence_after_sync();
    const long long ob = (b * Cs * O + outer) * SN + p;
#pragma unroll
    for (int c0 = 0; c0 < CX; c0 += 16) {
      if (c0 < Cs) {
        uint32_t dv[16];
        tc::tmem_ld16(tbase + lane_off + e.dcol + c0, dv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int o = c0 + i;
          if (o < Cs) {
            float val = __uint_as_float(dv[i]);
            const long long oi = ob + (long long)o * O * SN;
            if (MODE == EPI_BLOCK_FWD) {
              val += bias_s[o];
              if (pre_out) pre_out[oi] = from_f<T>(val);
              if (a.act) val = gelu_f(val);
            } else if (MODE == EPI_SPEC_BWD && a.tanh_pre) {
              const float th = tanhf(ldf<T>(x + oi));
              val *= 1.f - th * th;
            }
            out[oi] = from_f<T>(val);
          }
        }
      }
    }
    tc::fence_before_sync();
    if (__syncthreads_or(!ok)) break;   // B / A / D are rewritten by the next tile
  }
  if (!ok) tc::mbar_wait(mbar, phase & 1, nullptr);   // best effort: let in-flight MMAs land
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, TMEM_COLS);
}

// U[b, c, outer, r, k] = sum_q Z[b, c, outer, q, k] exp(+2 pi i kS(q) r / S)
__global__ void __launch_bounds__(256) k_inv_slab(const float2 *__restrict__ Z,
                                                  float2 *__restrict__ U, int S, int mS, int QS,
                                                  int mL) {
  extern __shared__ __align__(1024) unsigned char smem[];
  float2 *twS = reinterpret_cast<float2 *>(smem);
  float2 *zs = twS + S;                      // [QS][mL]
  const long long slab = blockIdx.x;
  build_twiddles(twS, S);
  const float2 *z = Z + slab * QS * mL;
  for (int i = threadIdx.x; i < QS * mL; i += blockDim.x) zs[i] = z[i];
  __syncthreads();
  float2 *u = U + slab * (long long)S * mL;
  for (int i = threadIdx.x; i < S * mL; i += blockDim.x) {
    const int r = i / mL, k = i - r * mL;
    float2 s = make_float2(0.f, 0.f);
    for (int q = 0; q < QS; ++q) {
      const int ks = QS == 1 ? 0 : kept_k(q, mS, S);
      cfma(s, zs[q * mL + k], twS[(int)(((long long)ks * r) % S)]);
    }
    u[i] = s;
  }
}

template <typename T, int MODE>
cudaError_t launch_epi_tc_m(const Launch &L, const Geom &g, const EpiTcArgs &a, int grid) {
  const int cmax = MODE == EPI_SPEC_BWD ? a.Ci : a.Co;
  const EpiTcGeom e = epi_tc_geom(g, MODE, a.Ci, a.Co, EKind<T>::EB, EKind<T>::tf32);
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)e.total);
    kern<<<grid, TC_THREADS, e.total, L.stream>>>(a, g);
  };
  if (cmax <= 16) go(k_epi_tc<T, MODE, 16>);
  else if (cmax <= 32) go(k_epi_tc<T, MODE, 32>);
  else go(k_epi_tc<T, MODE, 64>);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_epi_tc_t(const Launch &L, const Geom &g, int mode, const EpiTcArgs &a,
                            int grid) {
  if (mode == EPI_SPEC) return launch_epi_tc_m<T, EPI_SPEC>(L, g, a, grid);
  if (mode == EPI_BLOCK_FWD) return launch_epi_tc_m<T, EPI_BLOCK_FWD>(L, g, a, grid);
  return launch_epi_tc_m<T, EPI_SPEC_BWD>(L, g, a, grid);
}

}  // namespace

bool epi_tc_supported(const Geom &g, int dtype, int mode, int Ci, int Co) {
  if (mode == EPI_BLOCK_BWD) return false;
  if (!(g.NL % 128 == 0 || 128 % g.NL == 0)) return false;
  const long long SN = (long long)g.S * g.NL;
  if (SN % 128 != 0) return false;
  const bool tf32 = dtype == DT_F32;
  const EpiTcGeom e = epi_tc_geom(g, mode, Ci, Co, tf32 ? 4 : 2, tf32);
  if (e.dcol + e.NP > TMEM_COLS) return false;
  return e.total <= 227 * 1024;
}

size_t inv_slab_bytes(const Geom &g, long long C) {
  return sizeof(float2) * (size_t)(g.B * C * g.O) * g.S * g.mL;
}

cudaError_t launch_inv_slab(const Launch &L, const Geom &g, long long C, const float2 *Z,
                            float2 *U) {
  const long long slabs = g.B * C * g.O;
  const size_t smem = sizeof(float2) * ((size_t)g.S + (size_t)g.QS * g.mL);
  launch_begin(L);
  k_inv_slab<<<(unsigned)slabs, 256, smem, L.stream>>>(Z, U, g.S, g.mS, g.QS, g.mL);
  launch_end(L, "inv_slab");
  return cudaGetLastError();
}

cudaError_t launch_epilogue_tc(const Launch &L, const Geom &g, int dtype, int mode,
                               const EpiArgs &ea, const float2 *U) {
  EpiTcArgs a{};
  a.U = U;
  a.x = ea.x;
  a.W = ea.W;
  a.bias = ea.bias;
  a.out = ea.out;
  a.pre_out = ea.pre_out;
  a.err = L.err;
  a.Ci = ea.Ci;
  a.Co = ea.Co;
  a.act = ea.act;
  a.tanh_pre = ea.tanh_pre;
  const long long ntiles = g.B * g.O * ((long long)g.S * g.NL / TC_THREADS);
  const long long cap = 2LL * L.num_sms;
  const int grid = (int)(ntiles < cap ? ntiles : cap);
  static const char *const tags[3] = {"epi_spec_tc", "epi_block_fwd_tc", "epi_spec_bwd_tc"};
  launch_begin(L);
  cudaError_t err = dtype == DT_F32   ? launch_epi_tc_t<float>(L, g, mode, a, grid)
                    : dtype == DT_F16 ? launch_epi_tc_t<__half>(L, g, mode, a, grid)
                                      : launch_epi_tc_t<__nv_bfloat16>(L, g, mode, a, grid);
  launch_end(L, tags[mode < 3 ? mode : 2]);
  return err;
}

}  // namespace fno
