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

constexpr int TC_THREADS = 128;   // tile rows = TMEM lanes
constexpr int EPI_THREADS = 256;  // two warps per TMEM lane quarter, splitting channel groups
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

constexpr int UMAX = 16;   // spectrum values per thread per tile (B operand)

// Tile plan.  TMEM columns: D [0, NP); then the spectral A block of each
// last-axis tile offset ("variant"), resident for the whole kernel; then the
// x block, restaged per tile.  tf32 keeps hi and lo copies of both blocks.
struct EpiTcGeom {
  int Rt;        // slab rows per tile (NL < 128) or 1
  int nvar;      // distinct tile offsets along the last axis
  int KS, KSp;   // spectral K and its 16-padded width
  int KXp, KA, NP;
  int DC;        // TMEM columns of D: tf32 keeps A B_hi and A B_lo side by side (2 NP)
  int cs_cols;   // TMEM columns of one spectral variant (hi + lo)
  int x_col;     // first TMEM column of the x block
  int total_cols;
  int upt;       // spectrum values each thread loads per tile
  size_t bhi, blo, twL, bias, mbar, tbase, total;
  uint32_t sbo;
};

__host__ __device__ inline EpiTcGeom epi_tc_geom(const Geom &g, int mode, int Ci, int Co, int eb,
                                                 bool tf32) {
  EpiTcGeom e;
  e.Rt = g.NL >= 128 ? 1 : 128 / g.NL;
  e.nvar = g.NL >= 128 ? g.NL / 128 : 1;
  e.KS = e.Rt * 2 * g.mL;
  e.KSp = rup(e.KS, 16);
  e.KXp = mode == EPI_BLOCK_FWD ? rup(Ci, 16) : 0;
  e.KA = e.KSp + e.KXp;
  const int cs = (mode == EPI_SPEC_BWD) ? Ci : Co;
  e.NP = rup(cs, 16);
  e.DC = tf32 ? 2 * e.NP : e.NP;
  e.cs_cols = tf32 ? 2 * e.KSp : e.KSp / 2;
  e.x_col = e.DC + e.nvar * e.cs_cols;
  e.total_cols = e.x_col + (tf32 ? 2 * e.KXp : e.KXp / 2);
  e.upt = (e.Rt * cs * g.mL + 127) / 128;
  e.sbo = (uint32_t)(e.KA * eb / 16) * 128u;
  // B rows [0, NP) hold the hi split and rows [NP, 2 NP) the lo split (tf32), so
  // one MMA of width 2 NP applies both
  size_t off = 0;
  const size_t bbytes = (size_t)e.NP * e.KA * eb;
  e.bhi = off;
  e.blo = off + bbytes;
  off = al16(off + (tf32 ? 2 : 1) * bbytes);
  e.twL = off; off = al16(off + sizeof(float2) * g.NL);
  e.bias = off; off = al16(off + sizeof(float) * 64);
  e.mbar = off; off = al16(off + sizeof(uint64_t));
  e.tbase = off; off = al16(off + sizeof(uint32_t));
  e.total = off < 80 * 1024 ? 80 * 1024 : off;   // at most two CTAs per SM (TMEM)
  return e;
}

// byte offset of element (n, k) in a K-major no-swizzle B operand
__host__ __device__ __forceinline__ uint32_t boff(int n, int k, int eb, uint32_t sbo) {
  const int kb = k * eb;
  return (uint32_t)(n >> 3) * sbo + (kb >> 4) * 128 + (n & 7) * 16 + (kb & 15);
}

template <typename T>
__device__ __forceinline__ void bstore_at(unsigned char *bhi, unsigned char *blo, uint32_t o,
                                          float v) {
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

// stage 16 A elements into TMEM: tf32 -> hi at col, lo at col + lo_off;
// 16-bit -> 8 packed columns at col
template <typename T>
__device__ __forceinline__ void stage16(uint32_t col, uint32_t lo_off, const float (&v)[16]) {
  if (EKind<T>::tf32) {
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) tc::split_tf32(v[i], hi[i], lo[i]);
    tc::tmem_st16(col, hi);
    tc::tmem_st16(col + lo_off, lo);
  } else {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      pk[i] = EKind<T>::fmt == tc::FMT_BF16 ? tc::pack_bf16(v[2 * i], v[2 * i + 1])
                                             : tc::pack_f16(v[2 * i], v[2 * i + 1]);
    tc::tmem_st8(col, pk);
  }
}

template <typename T, int MODE, int CX>
__global__ void __launch_bounds__(EPI_THREADS) k_epi_tc(EpiTcArgs a, Geom g) {
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
  const int tid = threadIdx.x, warp = tid >> 5;
  const int t = tid & (TC_THREADS - 1);   // tile row (point) = TMEM lane
  const int half = tid >> 7;              // channel groups g with g % 2 == half
  const int NL = g.NL, S = g.S, mL = g.mL, O = g.O;
  const int Cs = MODE == EPI_SPEC_BWD ? Ci : Co;     // spectral output channels
  const long long SN = (long long)S * NL;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, TMEM_COLS);
    tc::tmem_relinquish();
  }
  if (tid == 0) tc::mbar_init(mbar, 1);
  build_twiddles(twL, NL);
  {  // B: zero, then W in columns [KSp, KSp + Ci)
    const size_t bbytes = (size_t)e.NP * e.KA * K::EB * (K::tf32 ? 2 : 1);
    for (size_t i = tid * 16; i < bbytes; i += EPI_THREADS * 16)
      *reinterpret_cast<uint4 *>(bhi + i) = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  if (MODE == EPI_BLOCK_FWD) {
    const T *W = reinterpret_cast<const T *>(a.W);
    for (int i = tid; i < Co * Ci; i += EPI_THREADS)
      bstore_at<T>(bhi, blo, boff(i / Ci, e.KSp + i % Ci, K::EB, e.sbo), to_f<T>(W[i]));
    const T *bias = reinterpret_cast<const T *>(a.bias);
    for (int o = tid; o < Co; o += EPI_THREADS) bias_s[o] = bias ? to_f<T>(bias[o]) : 0.f;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t arow = tbase + lane_off;
  const uint32_t lo_spec = K::tf32 ? (uint32_t)e.KSp : 0u;   // lo copy offset (columns)
  const uint32_t lo_x = K::tf32 ? (uint32_t)e.KXp : 0u;

  // resident spectral A block per variant: row t = point n0 + t (NL >= 128) or
  // point t of the Rt rows (NL < 128): (cos, -sin)(2 pi k n / NL) in the slot
  // of the point's row, zeros elsewhere
  for (int v = 0; v < e.nvar; ++v) {
    const int n = e.Rt > 1 ? t % NL : v * 128 + t;
    const int rl = e.Rt > 1 ? t / NL : 0;
    const uint32_t c0v = arow + e.DC + v * e.cs_cols;
    int r = 0, k = 0, par = 0, idx = 0;
    for (int c0 = 0; c0 < e.KSp; c0 += 16) {
      float vals[16];
      const bool mine = ((c0 >> 4) & 1) == half;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float val = 0.f;
        if (c0 + i < e.KS) {
          if (r == rl) {
            const float2 w = twL[idx];
            val = par ? -w.y : w.x;
          }
          if (par) {
            ++k;
            idx += n;
            if (idx >= NL) idx -= NL;
            if (k == mL) {
              k = 0;
              ++r;
              idx = 0;
            }
          }
          par ^= 1;
        }
        vals[i] = val;
      }
      if (mine) stage16<T>(c0v + (K::tf32 ? c0 : c0 / 2), lo_spec, vals);
    }
  }
  tc::tmem_wait_st();

  // this thread's share of the B spectral block: element i = t + 128 j of the
  // tile's [Rt][Cs][mL] spectrum, its offset inside the tile's U rows and its
  // smem position (row o, column r 2 mL + 2 k)
  int u_off[UMAX / 2];
  uint32_t b_off[UMAX / 2];
  float u_bias[UMAX / 2];   // bias added to the k = 0 real column (basis cos 0 = 1)
#pragma unroll
  for (int j = 0; j < UMAX / 2; ++j) {
    const int i = tid + EPI_THREADS * j;
    u_off[j] = -1;
    b_off[j] = 0;
    u_bias[j] = 0.f;
    if (i < e.Rt * Cs * mL) {
      const int k = i % mL, rest = i / mL;
      const int o = rest % Cs, r = rest / Cs;
      u_off[j] = (o * O * S + r) * mL + k;
      b_off[j] = boff(o, r * 2 * mL + 2 * k, K::EB, e.sbo);
      if (MODE == EPI_BLOCK_FWD && k == 0) u_bias[j] = bias_s[o];
    }
  }

  const T *x = reinterpret_cast<const T *>(a.x);
  T *out = reinterpret_cast<T *>(a.out);
  T *pre_out = reinterpret_cast<T *>(a.pre_out);
  const uint32_t idesc = tc::instr_desc(K::fmt, 128, e.DC);
  const uint64_t bdesc0 = tc::smem_desc_kmajor(tc::smem_u32(bhi), 128, e.sbo);
  const long long cstride = (long long)O * SN;     // channel stride of activations
  const int tps = (int)(SN / TC_THREADS);          // tiles per slab
  const long long ntiles = g.B * O * tps;
  const long long per_cta = (ntiles + gridDim.x - 1) / gridDim.x;
  const long long t_begin = blockIdx.x * per_cta;
  const long long t_end = t_begin + per_cta < ntiles ? t_begin + per_cta : ntiles;

  // Tile cursor: tiles of a CTA are consecutive, so (b, outer, row0, n0) is
  // advanced incrementally (no 64-bit division per tile).
  struct Cursor {
    long long b;
    int outer, row0, n0;   // first row of the tile and its last-axis offset
  };
  Cursor cur{0, 0, 0, 0};
  if (t_begin < t_end) {
    const long long slab = t_begin / tps;
    const int pb = (int)(t_begin - slab * tps) * TC_THREADS;
    cur.b = slab / O;
    cur.outer = (int)(slab - cur.b * O);
    cur.row0 = pb / NL;
    cur.n0 = pb - cur.row0 * NL;
  }
  auto advance = [&](Cursor c) {
    if (NL >= TC_THREADS) {
      c.n0 += TC_THREADS;
      if (c.n0 == NL) { c.n0 = 0; ++c.row0; }
    } else {
      c.row0 += e.Rt;
    }
    if (c.row0 == S) {
      c.row0 = 0;
      if (++c.outer == O) { c.outer = 0; ++c.b; }
    }
    return c;
  };

  constexpr int GPH = CX / 32 > 0 ? CX / 32 : 1;   // channel groups (of 16) per half
  float xr[GPH * 16];
  float2 ur[UMAX / 2];
  auto fetch = [&](const Cursor &c) {
    const long long pt = (long long)c.row0 * NL + c.n0 + t;
    if (MODE == EPI_BLOCK_FWD) {
      const T *xp = x + (c.b * Ci * O + c.outer) * SN + pt;
#pragma unroll
      for (int gi = 0; gi < GPH; ++gi) {
        const int c0 = (2 * gi + half) * 16;
        const T *xq = xp + (long long)c0 * cstride;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          xr[gi * 16 + i] = c0 + i < Ci ? ldf<T>(xq) : 0.f;
          xq += cstride;
        }
      }
    }
    const float2 *up = a.U + ((c.b * Cs * O + c.outer) * S + c.row0) * (long long)mL;
#pragma unroll
    for (int j = 0; j < UMAX / 2; ++j)
      if (u_off[j] >= 0) ur[j] = __ldg(up + u_off[j]);
  };

  uint32_t phase = 0;
  bool ok = true;
  if (t_begin < t_end) fetch(cur);
  for (long long tile = t_begin; tile < t_end; ++tile) {
    const Cursor c = cur;
    const bool new_rows = tile == t_begin || NL < TC_THREADS || c.n0 == 0;
    const int variant = e.Rt > 1 ? 0 : c.n0 / TC_THREADS;
    // (1) B spectral block (only when the tile's rows change)
    if (new_rows) {
#pragma unroll
      for (int j = 0; j < UMAX / 2; ++j) {
        if (u_off[j] >= 0) {
          bstore_at<T>(bhi, blo, b_off[j], ur[j].x + u_bias[j]);
          bstore_at<T>(bhi, blo, b_off[j] + K::EB, ur[j].y);
        }
      }
    }
    // (2) x block of A
    if (MODE == EPI_BLOCK_FWD) {
      const uint32_t xc = arow + e.x_col;
#pragma unroll
      for (int gi = 0; gi < GPH; ++gi) {
        const int c0 = (2 * gi + half) * 16;
        if (c0 < e.KXp) {
          float vals[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) vals[i] = xr[gi * 16 + i];
          stage16<T>(xc + (K::tf32 ? c0 : c0 / 2), lo_x, vals);
        }
      }
    }
    tc::tmem_wait_st();
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    // (3) one elected thread of warp 0 issues the MMAs: spectral K steps then x
    // K steps; for tf32 each K step is A_hi [B_hi; B_lo] + A_lo [B_hi; B_lo]
    if ((tid >> 5) == 0 && tc::elect_one()) {
      tc::fence_after_sync();
      const uint32_t aspec = tbase + e.DC + variant * e.cs_cols;
      const uint32_t ax = tbase + e.x_col;
      const int ns = e.KSp / K::KSTEP, nx = e.KXp / K::KSTEP;
      uint64_t bd = bdesc0;            // +256 bytes (16 units) per K step
      uint32_t acol = aspec;
#pragma unroll 4
      for (int s = 0; s < ns; ++s) {
        if (K::tf32) {
          tc::mma_tf32_ts(tbase, acol, bd, idesc, s > 0 ? 1u : 0u);
          tc::mma_tf32_ts(tbase, acol + lo_spec, bd, idesc, 1u);
        } else {
          tc::mma_f16_ts(tbase, acol, bd, idesc, s > 0 ? 1u : 0u);
        }
        bd += 16;
        acol += 8;
      }
      acol = ax;
#pragma unroll 4
      for (int s = 0; s < nx; ++s) {
        if (K::tf32) {
          tc::mma_tf32_ts(tbase, acol, bd, idesc, (ns + s) > 0 ? 1u : 0u);
          tc::mma_tf32_ts(tbase, acol + lo_x, bd, idesc, 1u);
        } else {
          tc::mma_f16_ts(tbase, acol, bd, idesc, (ns + s) > 0 ? 1u : 0u);
        }
        bd += 16;
        acol += 8;
      }
      tc::mma_commit(mbar);
    }
    // (4) prefetch the next tile while the MMAs run
    if (tile + 1 < t_end) {
      cur = advance(c);
      fetch(cur);
    }
    // (5) epilogue
    ok = tc::mbar_wait(mbar, phase & 1, a.err);
    phase++;
    tc::fence_after_sync();
    const long long ob = (c.b * Cs * O + c.outer) * SN + (long long)c.row0 * NL + c.n0 + t;
#pragma unroll
    for (int gi = 0; gi < GPH; ++gi) {
      const int c0 = (2 * gi + half) * 16;
      if (c0 < Cs) {
        uint32_t dv[16];
        tc::tmem_ld16(arow + c0, dv);
        float v[16];
        if (K::tf32) {
          uint32_t dl[16];
          tc::tmem_ld16(arow + e.NP + c0, dl);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; i += 2)
            f2unpack(f2add(f2pack(__uint_as_float(dv[i]), __uint_as_float(dv[i + 1])),
                           f2pack(__uint_as_float(dl[i]), __uint_as_float(dl[i + 1]))),
                     v[i], v[i + 1]);
        } else {
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(dv[i]);
        }
        const int nv = Cs - c0 < 16 ? Cs - c0 : 16;
        T *op = out + ob + (long long)c0 * cstride;
        if (MODE == EPI_BLOCK_FWD) {
          if (pre_out) {
            T *pp = pre_out + ob + (long long)c0 * cstride;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (i < nv) *pp = from_f<T>(v[i]);
              pp += cstride;
            }
          }
          if (a.act) {
#pragma unroll
            for (int i = 0; i < 16; i += 2) gelu2(v[i], v[i + 1]);
          }
        } else if (MODE == EPI_SPEC_BWD && a.tanh_pre) {
          const T *xq = x + ob + (long long)c0 * cstride;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (i < nv) {
              const float th = tanhf(ldf<T>(xq));
              v[i] *= 1.f - th * th;
            }
            xq += cstride;
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (i < nv) *op = from_f<T>(v[i]);
          op += cstride;
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
// One CTA per (b, c, outer) slab; a thread owns one row r and four modes.
__global__ void __launch_bounds__(256) k_inv_slab(const float2 *__restrict__ Z,
                                                  float2 *__restrict__ U, int S, int mS, int QS,
                                                  int mL) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int mLp = (mL + 3) & ~3;
  float2 *twS = reinterpret_cast<float2 *>(smem);
  float2 *zs = twS + ((S + 1) & ~1);          // [QS][mLp], 16-byte aligned rows
  const long long slab = blockIdx.x;
  build_twiddles(twS, S);
  const float2 *z = Z + slab * QS * mL;
  for (int i = threadIdx.x; i < QS * mLp; i += blockDim.x) {
    const int q = i / mLp, k = i - q * mLp;
    zs[i] = k < mL ? z[q * mL + k] : make_float2(0.f, 0.f);
  }
  __syncthreads();
  float2 *u = U + slab * (long long)S * mL;
  const int mLg = mLp / 4;
  for (int i = threadIdx.x; i < S * mLg; i += blockDim.x) {
    const int r = i / mLg, kg = i - r * mLg;
    float2 acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] = make_float2(0.f, 0.f);
    KeptIndex ki(QS == 1 ? 0 : mS, S, r);
    for (int q = 0; q < QS; ++q) {
      const float2 w = twS[ki.next()];
      const float4 z01 = *reinterpret_cast<const float4 *>(zs + q * mLp + 4 * kg);
      const float4 z23 = *reinterpret_cast<const float4 *>(zs + q * mLp + 4 * kg + 2);
      cfma(acc[0], make_float2(z01.x, z01.y), w);
      cfma(acc[1], make_float2(z01.z, z01.w), w);
      cfma(acc[2], make_float2(z23.x, z23.y), w);
      cfma(acc[3], make_float2(z23.z, z23.w), w);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (4 * kg + j < mL) u[r * mL + 4 * kg + j] = acc[j];
  }
}

template <typename T, int MODE>
cudaError_t launch_epi_tc_m(const Launch &L, const Geom &g, const EpiTcArgs &a, int grid) {
  const int cmax = MODE == EPI_SPEC_BWD ? a.Ci : a.Co;
  const EpiTcGeom e = epi_tc_geom(g, MODE, a.Ci, a.Co, EKind<T>::EB, EKind<T>::tf32);
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)e.total);
    kern<<<grid, EPI_THREADS, e.total, L.stream>>>(a, g);
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
  if (e.total_cols > TMEM_COLS || e.DC > 256) return false;
  if (e.Rt * ((mode == EPI_SPEC_BWD) ? Ci : Co) * g.mL > (UMAX / 2) * EPI_THREADS) return false;
  return e.total <= 227 * 1024;
}

size_t inv_slab_bytes(const Geom &g, long long C) {
  return sizeof(float2) * (size_t)(g.B * C * g.O) * g.S * g.mL;
}

cudaError_t launch_inv_slab(const Launch &L, const Geom &g, long long C, const float2 *Z,
                            float2 *U) {
  const long long slabs = g.B * C * g.O;
  const size_t smem = sizeof(float2) * ((size_t)((g.S + 1) & ~1) + (size_t)g.QS * ((g.mL + 3) & ~3));
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
