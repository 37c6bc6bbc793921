// Forward truncated transform (steps S0-S2) on the sm_100a tensor cores.
//
// S1, the last-axis DFT, is the dense contraction
//     X1[row, j] = sum_n s[row, n] F[j, n],   F[2k] = cos(2 pi k n / N_L),
//                                             F[2k+1] = -sin(2 pi k n / N_L),
// with rows = (b, c, outer, slab row).  A CTA takes 128 consecutive rows
// (M = 128, thread t <-> row t <-> TMEM lane t), streams each row through
// registers in 128-byte chunks (applying tanh or the GELU derivative on the
// way), and writes it into tensor memory as the MMA's A operand; F is the B
// operand, built once per CTA in shared memory.  For float32 storage the
// product is taken in three tf32 passes, A_hi F_hi + A_hi F_lo + A_lo F_hi,
// with hi = tf32(x), lo = tf32(x - hi), which keeps ~21 bits; 16-bit storage
// uses one kind::f16 pass with float32 accumulation.
//
// S2, the slab-axis contraction X2[q, k] = sum_r X1[r, k] exp(-i theta_S(q, r)),
// runs on the CUDA cores from a shared-memory copy of the tile's X1.  Tiles
// that cover a whole slab write it complete; tiles of a longer slab write a
// partial sum per 128-row band, which the finishing kernel adds.
#include "fno_common.cuh"
#include "fno_kernels.cuh"
#include "tc_util.cuh"

namespace fno {

namespace {

constexpr int TC_THREADS = 128;
constexpr int TMEM_COLS = 256;
constexpr int A_COL0 = 128;        // A buffers start here; D occupies [0, NP)

struct S1Args {
  const void *in0, *in1;
  float2 *zpart;        // [nbands][planes][QS][mL]
  int *err;
  long long planes, total_rows;
  int S, NL, mL, mS, QS, NP, nbands;
};

template <typename T> struct Kind {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int fmt = tc::FMT_F16;
};
template <> struct Kind<float> {
  static constexpr bool tf32 = true;
  static constexpr int EB = 4;
  static constexpr int fmt = tc::FMT_TF32;
};
template <> struct Kind<__nv_bfloat16> {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int fmt = tc::FMT_BF16;
};

struct S1Layout {
  size_t fhi, flo, twL, twS, x1, xs, mbar, tbase, total;
  int x1_ld, mLp;
};

constexpr int XS_LD = 144;   // bytes per staged row chunk (128 + 16 pad: conflict-free rows)

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~(size_t)15; }

__host__ __device__ inline S1Layout s1_layout(int S, int NL, int mL, int NP, int EB, bool tf32) {
  S1Layout l;
  l.mLp = (mL + 3) & ~3;
  l.x1_ld = 2 * l.mLp + 4;
  size_t off = 0;
  const size_t fbytes = (size_t)NP * NL * EB;
  l.fhi = off; off = al16(off + fbytes);
  l.flo = off; if (tf32) off = al16(off + fbytes);
  l.twL = off; off = al16(off + sizeof(float2) * NL);
  l.twS = off; off = al16(off + sizeof(float2) * S);
  // the staged row chunks (chunk loop) and the X1 copy (after it) share space
  const size_t x1b = sizeof(float) * (size_t)TC_THREADS * l.x1_ld;
  const size_t xsb = 2 * (size_t)TC_THREADS * XS_LD;
  l.x1 = off;
  l.xs = off;
  off = al16(off + (x1b > xsb ? x1b : xsb));
  l.mbar = off; off = al16(off + 2 * sizeof(uint64_t));
  l.tbase = off; off = al16(off + sizeof(uint32_t));
  // keep at most two CTAs per SM so their TMEM allocations always fit
  l.total = off < 80 * 1024 ? 80 * 1024 : off;
  return l;
}

template <typename T>
__device__ __forceinline__ float elem(const uint4 (&raw)[8], int i) {
  if (sizeof(T) == 4) {
    const uint32_t *u = reinterpret_cast<const uint32_t *>(raw);
    return __uint_as_float(u[i]);
  } else {
    const T *h = reinterpret_cast<const T *>(raw);
    return to_f<T>(h[i]);
  }
}

// apply the load transform (tanh, or dz = dy * GELU'(pre)) to one 16-byte
// piece, keeping the storage format
template <typename T, int LOAD>
__device__ __forceinline__ uint4 transform16(uint4 v0, uint4 v1) {
  if (LOAD == LOAD_PLAIN) return v0;
  constexpr int NE = 16 / sizeof(T);
  T *a = reinterpret_cast<T *>(&v0);
  const T *b = reinterpret_cast<const T *>(&v1);
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    float x = to_f<T>(a[i]);
    if (LOAD == LOAD_TANH) x = tanhf(x);
    if (LOAD == LOAD_DZ) x *= gelu_grad_f(to_f<T>(b[i]));
    a[i] = from_f<T>(x);
  }
  return v0;
}

template <typename T, int LOAD>
__global__ void __launch_bounds__(TC_THREADS) k_s1_tc(S1Args a) {
  using K = Kind<T>;
  constexpr int EB = K::EB;
  constexpr int CW = 128 / EB;              // elements per 128-byte chunk
  constexpr int ACOLS = K::tf32 ? 64 : 32;  // TMEM columns per A buffer
  extern __shared__ __align__(1024) unsigned char smem[];
  const int NL = a.NL, S = a.S, mL = a.mL, QS = a.QS, NP = a.NP;
  const S1Layout lay = s1_layout(S, NL, mL, NP, EB, K::tf32);
  unsigned char *fhi = smem + lay.fhi;
  unsigned char *flo = smem + lay.flo;
  float2 *twL = reinterpret_cast<float2 *>(smem + lay.twL);
  float2 *twS = reinterpret_cast<float2 *>(smem + lay.twS);
  float *x1s = reinterpret_cast<float *>(smem + lay.x1);
  uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + lay.mbar);
  uint32_t *tbase_s = reinterpret_cast<uint32_t *>(smem + lay.tbase);
  unsigned char *xs = smem + lay.xs;       // [2][128][XS_LD] staged row chunks
  const int t = threadIdx.x, warp = t >> 5;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (t == 0) {
    tc::mbar_init(&mbar[0], 1);
    tc::mbar_init(&mbar[1], 1);
  }
  build_twiddles(twL, NL);
  build_twiddles(twS, S);
  __syncthreads();
  // B operand F[j][n] (j < NP rows, n < NL), K-major core-matrix layout
  const uint32_t sbo = (uint32_t)(NL * EB / 16) * 128u;
  for (int e = t; e < NP * NL; e += TC_THREADS) {
    const int j = e / NL, n = e - j * NL;
    float v = 0.f;
    if (j < 2 * mL) {
      const float2 w = twL[((j >> 1) * n) % NL];
      v = (j & 1) ? -w.y : w.x;
    }
    const int kb = n * EB;
    const size_t off = (size_t)(j >> 3) * sbo + (kb >> 4) * 128 + (j & 7) * 16 + (kb & 15);
    if (K::tf32) {
      uint32_t hi, lo;
      tc::split_tf32(v, hi, lo);
      *reinterpret_cast<uint32_t *>(fhi + off) = hi;
      *reinterpret_cast<uint32_t *>(flo + off) = lo;
    } else {
      *reinterpret_cast<T *>(fhi + off) = from_f<T>(v);
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  // tf32: F rows [0, NP) hold the hi split and [NP, 2 NP) the lo split (contiguous),
  // so A [F_hi; F_lo] is one MMA of width 2 NP; D keeps both halves
  const int DC = K::tf32 ? 2 * NP : NP;
  const uint32_t idesc = tc::instr_desc(K::fmt, 128, DC);
  const uint64_t fdesc0 = tc::smem_desc_kmajor(tc::smem_u32(fhi), 128, sbo);
  (void)flo;

  const T *in0 = reinterpret_cast<const T *>(a.in0);
  const T *in1 = reinterpret_cast<const T *>(a.in1);
  const int nchunks = NL / CW;
  const long long ntiles = (a.total_rows + TC_THREADS - 1) / TC_THREADS;
  uint32_t g = 0;      // chunks issued by this CTA (selects buffer and phase)
  bool ok = true;

  for (long long tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
    const long long row0 = tile * TC_THREADS;
    // coalesced loading: thread t fetches 16-byte piece (t & 7) of rows
    // (t >> 3) + 16 j, j < 8, for every 128-byte chunk of the row
    const int seg = t & 7;
    const uint4 *src0[8];
    const uint4 *src1[8];
    bool rv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const long long row = row0 + (t >> 3) + 16 * j;
      rv[j] = row < a.total_rows;
      const long long rr = rv[j] ? row : 0;
      src0[j] = reinterpret_cast<const uint4 *>(in0 + rr * NL) + seg;
      src1[j] = LOAD == LOAD_DZ ? reinterpret_cast<const uint4 *>(in1 + rr * NL) + seg : nullptr;
    }
    uint4 p0[8], p1[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      p0[j] = rv[j] ? __ldg(src0[j]) : make_uint4(0, 0, 0, 0);
      if (LOAD == LOAD_DZ) p1[j] = rv[j] ? __ldg(src1[j]) : make_uint4(0, 0, 0, 0);
    }
    for (int c = 0; c < nchunks; ++c, ++g) {
      const uint32_t buf = g & 1;
      unsigned char *xb = xs + buf * (TC_THREADS * XS_LD);
      // (1) transformed pieces of chunk c -> shared memory
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4 *>(xb + ((t >> 3) + 16 * j) * XS_LD + seg * 16) =
            transform16<T, LOAD>(p0[j], LOAD == LOAD_DZ ? p1[j] : p0[j]);
      // (2) prefetch chunk c + 1
      if (c + 1 < nchunks) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          p0[j] = rv[j] ? __ldg(src0[j] + (c + 1) * 8) : make_uint4(0, 0, 0, 0);
          if (LOAD == LOAD_DZ) p1[j] = rv[j] ? __ldg(src1[j] + (c + 1) * 8) : make_uint4(0, 0, 0, 0);
        }
      }
      // (3) the A buffer of chunk c - 2 must be free
      if (g >= 2) ok = tc::mbar_wait(&mbar[buf], ((g - 2) >> 1) & 1, a.err);
      if (__syncthreads_or(!ok)) { ok = false; break; }
      tc::fence_after_sync();
      // (4) this thread's row of the chunk -> A operand in TMEM
      uint4 r0[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) r0[v] = *reinterpret_cast<const uint4 *>(xb + t * XS_LD + v * 16);
      const uint32_t acol = tbase + lane_off + A_COL0 + buf * ACOLS;
#pragma unroll
      for (int h = 0; h < CW / 16; ++h) {      // 16 elements per step
        float xv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) xv[i] = elem<T>(r0, h * 16 + i);
        if (K::tf32) {
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) tc::split_tf32(xv[i], hi[i], lo[i]);
          tc::tmem_st16(acol + h * 16, hi);
          tc::tmem_st16(acol + 32 + h * 16, lo);
        } else {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = Kind<T>::fmt == tc::FMT_BF16 ? tc::pack_bf16(xv[2 * i], xv[2 * i + 1])
                                                  : tc::pack_f16(xv[2 * i], xv[2 * i + 1]);
          tc::tmem_st8(acol + h * 8, pk);
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncthreads();
      if ((t >> 5) == 0 && tc::elect_one()) {   // one elected thread of warp 0
        tc::fence_after_sync();
        const uint32_t a0 = tbase + A_COL0 + buf * ACOLS;
        // descriptors advance by constants (256 bytes = 16 units per K step)
        const uint64_t bh0 = fdesc0 + (uint64_t)(c * 4 * 16);
        const uint32_t acc0 = c ? 1u : 0u;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t bh = bh0 + (uint64_t)(s * 16);
          const uint32_t acc = s ? 1u : acc0;
          if (K::tf32) {
            tc::mma_tf32_ts(tbase, a0 + s * 8, bh, idesc, acc);
            tc::mma_tf32_ts(tbase, a0 + 32 + s * 8, bh, idesc, 1u);
          } else {
            tc::mma_f16_ts(tbase, a0 + s * 8, bh, idesc, acc);
          }
        }
        tc::mma_commit(&mbar[buf]);
      }
    }
    if (!ok) break;
    // all MMAs of the tile are done once the last chunk's commit has arrived
    const uint32_t gl = g - 1;
    ok = tc::mbar_wait(&mbar[gl & 1], (gl >> 1) & 1, a.err);
    if (__syncthreads_or(!ok)) { ok = false; break; }
    tc::fence_after_sync();
    // D row -> shared memory (row t, 2 mL floats)
    float *myx1 = x1s + t * lay.x1_ld;
    for (int c0 = 0; c0 < NP; c0 += 16) {
      uint32_t v[16];
      tc::tmem_ld16(tbase + lane_off + c0, v);
      if (K::tf32) {
        uint32_t vl[16];
        tc::tmem_ld16(tbase + lane_off + NP + c0, vl);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(vl[i]));
      } else {
        tc::tmem_wait_ld();
      }
#pragma unroll
      for (int i = 0; i < 16; i += 4) {
        if (c0 + i < 2 * lay.mLp)
          *reinterpret_cast<float4 *>(myx1 + c0 + i) =
              make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                          __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
      }
    }
    tc::fence_before_sync();
    __syncthreads();
    // S2: slab-axis contraction of the tile's rows
    const int rows_per_slab = S < TC_THREADS ? S : TC_THREADS;
    const int slabs = TC_THREADS / rows_per_slab;
    const int mLg = lay.mLp / 4;
    const int r_off = S < TC_THREADS ? 0 : (int)(row0 % S);
    const int band = S < TC_THREADS ? 0 : r_off / TC_THREADS;
    const long long plane0 = row0 / S;
    const int nout = slabs * QS * mLg;
    for (int e = t; e < nout; e += TC_THREADS) {
      const int kg = e % mLg;
      const int rest = e / mLg;
      const int q = rest % QS, si = rest / QS;
      const long long plane = plane0 + si;
      if (plane >= a.planes) continue;
      const int ks = QS == 1 ? 0 : kept_k(q, a.mS, S);
      float2 acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
      const float *xr = x1s + (si * rows_per_slab) * lay.x1_ld + kg * 8;
      int idx = mulmod(ks, r_off % S, S);
      int r = 0;
      for (; r + 4 <= rows_per_slab; r += 4) {     // four rows per step: loads ahead of FMAs
        float2 w[4];
        float4 p0[4], p1[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          w[u] = twS[idx];
          idx += ks;
          if (idx >= S) idx -= S;
          p0[u] = *reinterpret_cast<const float4 *>(xr + (r + u) * lay.x1_ld);
          p1[u] = *reinterpret_cast<const float4 *>(xr + (r + u) * lay.x1_ld + 4);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          cfma_conj_b(acc[0], make_float2(p0[u].x, p0[u].y), w[u]);
          cfma_conj_b(acc[1], make_float2(p0[u].z, p0[u].w), w[u]);
          cfma_conj_b(acc[2], make_float2(p1[u].x, p1[u].y), w[u]);
          cfma_conj_b(acc[3], make_float2(p1[u].z, p1[u].w), w[u]);
        }
      }
      for (; r < rows_per_slab; ++r) {
        const float2 w = twS[idx];
        idx += ks;
        if (idx >= S) idx -= S;
        const float4 p0 = *reinterpret_cast<const float4 *>(xr + r * lay.x1_ld);
        const float4 p1 = *reinterpret_cast<const float4 *>(xr + r * lay.x1_ld + 4);
        cfma_conj_b(acc[0], make_float2(p0.x, p0.y), w);
        cfma_conj_b(acc[1], make_float2(p0.z, p0.w), w);
        cfma_conj_b(acc[2], make_float2(p1.x, p1.y), w);
        cfma_conj_b(acc[3], make_float2(p1.z, p1.w), w);
      }
      float2 *dst = a.zpart + (((long long)band * a.planes + plane) * QS + q) * mL;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (kg * 4 + i < mL) dst[kg * 4 + i] = acc[i];
    }
    __syncthreads();  // x1s is rewritten by the next tile
  }
  // drain: no MMA of this CTA may still be reading TMEM when it is freed
  if (g > 0) {
    const uint32_t gl = g - 1;
    tc::mbar_wait(&mbar[gl & 1], (gl >> 1) & 1, a.err);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tbase, TMEM_COLS);
}

template <typename T>
cudaError_t launch_s1_t(const Launch &L, int load_mode, int grid, size_t smem, const S1Args &a) {
  auto set = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, TC_THREADS, smem, L.stream>>>(a);
  };
  if (load_mode == LOAD_PLAIN) set(k_s1_tc<T, LOAD_PLAIN>);
  else if (load_mode == LOAD_TANH) set(k_s1_tc<T, LOAD_TANH>);
  else set(k_s1_tc<T, LOAD_DZ>);
  return cudaGetLastError();
}

}  // namespace

// Shapes the tensor-core transform handles: whole 128-byte chunks per row,
// 128-row tiles that never split a slab unevenly, and a D accumulator of at
// most 128 columns.
bool s1_tc_supported(const Geom &g, int dtype) {
  const int eb = dtype == DT_F32 ? 4 : 2;
  if ((g.NL * eb) % 128 != 0) return false;
  if (!(g.S % 128 == 0 || 128 % g.S == 0)) return false;
  const int np = ((2 * g.mL + 15) / 16) * 16;
  if ((dtype == DT_F32 ? 2 * np : np) > 128) return false;   // D must fit below the A buffers
  const S1Layout l = s1_layout(g.S, g.NL, g.mL, np, eb, dtype == DT_F32);
  return l.total <= 227 * 1024;
}

int s1_tc_bands(const Geom &g) { return g.S >= 128 ? g.S / 128 : 1; }

cudaError_t launch_s1_tc(const Launch &L, const Geom &g, int dtype, int load_mode, long long C,
                         const void *in0, const void *in1, float2 *zpart, int *err) {
  S1Args a{};
  a.in0 = in0;
  a.in1 = in1;
  a.zpart = zpart;
  a.err = err;
  a.planes = g.B * C * g.O;
  a.total_rows = a.planes * g.S;
  a.S = g.S;
  a.NL = g.NL;
  a.mL = g.mL;
  a.mS = g.mS;
  a.QS = g.QS;
  a.NP = ((2 * g.mL + 15) / 16) * 16;
  a.nbands = s1_tc_bands(g);
  const int eb = dtype == DT_F32 ? 4 : 2;
  const S1Layout lay = s1_layout(g.S, g.NL, g.mL, a.NP, eb, dtype == DT_F32);
  const long long ntiles = (a.total_rows + TC_THREADS - 1) / TC_THREADS;
  const long long cap = 2LL * L.num_sms;
  const int grid = (int)(ntiles < cap ? ntiles : cap);
  launch_begin(L);
  cudaError_t err_ = dtype == DT_F32   ? launch_s1_t<float>(L, load_mode, grid, lay.total, a)
                     : dtype == DT_F16 ? launch_s1_t<__half>(L, load_mode, grid, lay.total, a)
                                       : launch_s1_t<__nv_bfloat16>(L, load_mode, grid, lay.total, a);
  launch_end(L, load_mode == LOAD_DZ ? "fwd_transform_tc_dz" : "fwd_transform_tc");
  return err_;
}

}  // namespace fno
