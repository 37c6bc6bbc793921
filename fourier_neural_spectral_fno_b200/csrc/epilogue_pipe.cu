// Fused block epilogue (step S4, forward) as a warp-specialised, TMA-fed
// tcgen05 pipeline.
//
// The arithmetic is the per-tile GEMM of the tensor-core epilogue: for a tile
// of 128 consecutive grid points of one (sample, outer index) slab
//     pre[p, o] = sum_j basis[p, j] U[o, j] + sum_i x[p, i] W[o, i] + b[o]
// with basis = (cos, -sin)(2 pi k n / N_L) of the point's last-axis index n
// and U the spectrum already inverted along the slab axis (k_inv_slab).  The
// difference is the schedule: every role runs in its own warps and the tiles
// stream through the SM, so HBM traffic, staging, MMAs and the GELU epilogue
// of consecutive tiles overlap.
//
//   warp 17       TMA producer: x tile [Ci][128] and U rows [Co][Rt 2 mL] of
//                 tile j into ring stage j % NS (mbarrier transaction count)
//   warps 0-7     staging: U -> B operand (smem, K-major core matrices,
//                 tf32 hi/lo split, bias folded into the k = 0 column), x ->
//                 A operand (TMEM, one lane per point); double-buffered; two
//                 warps per TMEM lane quarter, each owning half of the x
//                 channel groups and of the B chunks
//   warp 16       one thread issues the MMAs of tile j into D buffer j % 2
//   warps 8-15    epilogue: D -> registers, bias already in, optional pre
//                 store, GELU, coalesced y stores; two warps per TMEM lane
//                 quarter, each owning half of the channel groups
//
// Hand-offs (all mbarriers, every wait bounded):
//   full[s]   TMA -> staging (transaction bytes)   empty[s]  staging -> TMA
//   aready[i] staging -> MMA                       mdone[i]  MMA -> epilogue
//   dempty[i] epilogue -> MMA                      (mdone also frees A/B)
// A waiter never falls two phases behind its barrier: each barrier's next
// phase needs an action that follows the wait in program order.
#include <string.h>

#include "fno_common.cuh"
#include "fno_kernels.cuh"
#include "tc_util.cuh"
#include "tma_util.cuh"

namespace fno {

namespace {

constexpr int ROWS = 128;                  // points per tile = TMEM lanes
constexpr int NCONV = 8;                   // staging warps (two per TMEM lane quarter)
constexpr int NEPI = 8;                    // epilogue warps
constexpr int WARP_MMA = NCONV + NEPI;     // 16
constexpr int WARP_TMA = WARP_MMA + 1;     // 17
constexpr int THREADS = (WARP_TMA + 1) * 32;
constexpr int MAX_STAGES = 6;
constexpr size_t kSmemMax = 227 * 1024;

template <typename T> struct PKind {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int KSTEP = 16;
  static constexpr int fmt = tc::FMT_F16;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
};
template <> struct PKind<float> {
  static constexpr bool tf32 = true;
  static constexpr int EB = 4;
  static constexpr int KSTEP = 8;
  static constexpr int fmt = tc::FMT_TF32;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
};
template <> struct PKind<__nv_bfloat16> {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int KSTEP = 16;
  static constexpr int fmt = tc::FMT_BF16;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};

__host__ __device__ inline int rup(int v, int m) { return (v + m - 1) / m * m; }
__host__ __device__ inline size_t alg(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Tile plan.  TMEM columns: two D buffers [0, 2 DC), the resident spectral A
// block of every last-axis tile offset ("variant"), then NA x-blocks of A.
// Shared memory: NS ring stages (x tile, U rows), NA B buffers (hi rows then
// lo rows), the last-axis twiddles, the bias, mbarriers.
struct PipeGeom {
  int Rt, nvar, KS, KSp, KXp, KA, NP, DC, DA, cs_cols, ax_cols;
  int NA, NS, NB;
  int col_spec, col_x, used_cols, cols;
  uint32_t sbo, sbo_s, x_bytes, u_bytes;
  size_t uoff, stage, bhalf, bbuf, b, tw, bias, bar, tbase, total;
};

// img: the spectral half of B arrives prebuilt per grid row (the slab-axis
// inverse writes it in the operand layout), so the B buffer holds W alone
__host__ __device__ inline PipeGeom pipe_geom(const Geom &g, bool has_x, int Ci, int Co, int eb,
                                              bool tf32, bool img = false) {
  PipeGeom e;
  e.Rt = g.NL >= ROWS ? 1 : ROWS / g.NL;
  e.nvar = g.NL >= ROWS ? g.NL / ROWS : 1;
  e.KS = e.Rt * 2 * g.mL;
  e.KSp = rup(e.KS, 16);
  e.KXp = has_x ? rup(Ci, 16) : 0;
  e.KA = e.KSp + e.KXp;
  e.NP = rup(Co, 16);
  e.DC = tf32 ? 2 * e.NP : e.NP;           // rows of B (tf32: hi rows, then lo rows)
  e.DA = e.NP;                             // accumulator columns
  e.cs_cols = tf32 ? 2 * e.KSp : e.KSp / 2;
  e.ax_cols = tf32 ? 2 * e.KXp : e.KXp / 2;
  e.col_spec = 2 * e.DA;
  e.col_x = e.col_spec + e.nvar * e.cs_cols;
  e.NA = e.col_x + 2 * e.ax_cols <= 512 ? 2 : 1;
  e.used_cols = e.col_x + e.NA * e.ax_cols;
  e.cols = 32;
  while (e.cols < e.used_cols && e.cols < 1024) e.cols *= 2;
  const int kb = img ? e.KXp : e.KA;            // K of the B buffer
  e.sbo = (uint32_t)(kb * eb / 16) * 128u;
  e.sbo_s = (uint32_t)(e.KSp * eb / 16) * 128u;  // the prebuilt spectral image
  e.x_bytes = has_x ? (uint32_t)(Ci * ROWS * eb) : 0u;
  e.u_bytes = img ? (uint32_t)(e.DC * e.KSp * eb) : (uint32_t)(Co * e.KS * 4);
  e.uoff = alg(e.x_bytes, 128);
  e.stage = alg(e.uoff + e.u_bytes, 1024);
  e.bhalf = (size_t)e.NP * kb * eb;
  e.bbuf = alg((tf32 ? 2 : 1) * e.bhalf, 1024);
  e.NB = img ? 1 : e.NA;                         // W is constant: one buffer
  const size_t fixed = e.NB * e.bbuf + alg(sizeof(float2) * g.NL, 128) + sizeof(float) * 64 +
                       sizeof(uint64_t) * (2 * MAX_STAGES + 6) + 16;
  const size_t room = kSmemMax > fixed ? kSmemMax - fixed : 0;
  const size_t ns = room / e.stage;
  e.NS = (int)(ns < (size_t)MAX_STAGES ? ns : (size_t)MAX_STAGES);
  size_t off = 0;
  off += (size_t)(e.NS > 0 ? e.NS : 0) * e.stage;
  e.b = off; off += e.NB * e.bbuf;
  e.tw = off; off = alg(off + sizeof(float2) * g.NL, 128);
  e.bias = off; off += sizeof(float) * 64;
  e.bar = off; off += sizeof(uint64_t) * (2 * MAX_STAGES + 6);
  e.tbase = off; off += 16;
  // one CTA per SM: the TMEM allocation may take all 512 columns
  e.total = off < 116 * 1024 ? 116 * 1024 : off;
  return e;
}

// byte offset of element (n, k) in a K-major no-swizzle B operand
__host__ __device__ __forceinline__ uint32_t boff(int n, int k, int eb, uint32_t sbo) {
  const int kb = k * eb;
  return (uint32_t)(n >> 3) * sbo + (kb >> 4) * 128 + (n & 7) * 16 + (kb & 15);
}

template <typename T>
__device__ __forceinline__ void bstore1(unsigned char *bh, size_t bhalf, uint32_t o, float v) {
  if (PKind<T>::tf32) {
    uint32_t hi, lo;
    tc::split_tf32(v, hi, lo);
    *reinterpret_cast<uint32_t *>(bh + o) = hi;
    *reinterpret_cast<uint32_t *>(bh + bhalf + o) = lo;
  } else {
    *reinterpret_cast<T *>(bh + o) = from_f<T>(v);
  }
}

// four K-consecutive elements (k multiple of 4) in one store per half
template <typename T>
__device__ __forceinline__ void bstore4(unsigned char *bh, size_t bhalf, uint32_t o, float4 v) {
  if (PKind<T>::tf32) {
    uint32_t h0, h1, h2, h3, l0, l1, l2, l3;
    tc::split_tf32(v.x, h0, l0);
    tc::split_tf32(v.y, h1, l1);
    tc::split_tf32(v.z, h2, l2);
    tc::split_tf32(v.w, h3, l3);
    *reinterpret_cast<uint4 *>(bh + o) = make_uint4(h0, h1, h2, h3);
    *reinterpret_cast<uint4 *>(bh + bhalf + o) = make_uint4(l0, l1, l2, l3);
  } else if (PKind<T>::fmt == tc::FMT_BF16) {
    *reinterpret_cast<uint2 *>(bh + o) = make_uint2(tc::pack_bf16(v.x, v.y), tc::pack_bf16(v.z, v.w));
  } else {
    *reinterpret_cast<uint2 *>(bh + o) = make_uint2(tc::pack_f16(v.x, v.y), tc::pack_f16(v.z, v.w));
  }
}

// 16 A elements of this thread's lane into TMEM (tf32: hi at col, lo at col + lo_off)
template <typename T>
__device__ __forceinline__ void stage16(uint32_t col, uint32_t lo_off, const float (&v)[16]) {
  if (PKind<T>::tf32) {
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) tc::split_tf32(v[i], hi[i], lo[i]);
    tc::tmem_st16(col, hi);
    tc::tmem_st16(col + lo_off, lo);
  } else {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      pk[i] = PKind<T>::fmt == tc::FMT_BF16 ? tc::pack_bf16(v[2 * i], v[2 * i + 1])
                                             : tc::pack_f16(v[2 * i], v[2 * i + 1]);
    tc::tmem_st8(col, pk);
  }
}

struct PipeArgs {
  const void *W, *bias;
  void *out, *pre_out;
  const unsigned char *img;   // prebuilt spectral B images per grid row (IMG), else NULL
  int *err;
  int Ci, Co, act;
};

// tile cursor (tiles of a CTA are consecutive)
struct Cursor {
  long long b;
  int outer, row0, n0;
};

__device__ __forceinline__ Cursor cursor_at(long long tile, int tps, const Geom &g) {
  Cursor c{0, 0, 0, 0};
  const long long slab = tile / tps;
  const int pb = (int)(tile - slab * tps) * ROWS;
  c.b = slab / g.O;
  c.outer = (int)(slab - c.b * g.O);
  c.row0 = pb / g.NL;
  c.n0 = pb - c.row0 * g.NL;
  return c;
}

__device__ __forceinline__ void cursor_next(Cursor &c, int Rt, const Geom &g) {
  if (g.NL >= ROWS) {
    c.n0 += ROWS;
    if (c.n0 == g.NL) {
      c.n0 = 0;
      ++c.row0;
    }
  } else {
    c.row0 += Rt;
  }
  if (c.row0 == g.S) {
    c.row0 = 0;
    if (++c.outer == g.O) {
      c.outer = 0;
      ++c.b;
    }
  }
}

// NSTEP K steps of the tile's MMA chain into D, unrolled: every operand is a
// base plus a compile-time offset (8 TMEM columns of A, 256 bytes of B per
// step).  acc_first: the first step accumulates onto D as well.
template <typename K, int NSTEP>
__device__ __forceinline__ void issue_exact(uint32_t d, uint32_t a, uint32_t lo, uint64_t b,
                                            uint64_t blo, uint32_t idesc, bool acc_first) {
#pragma unroll
  for (int s = 0; s < NSTEP; ++s) {
    const uint32_t acc = (acc_first || s > 0) ? 1u : 0u;
    if (K::tf32) {   // A_hi B_hi + A_lo B_hi + A_hi B_lo
      tc::mma_tf32_ts(d, a + 8 * s, b + (uint64_t)(16 * s), idesc, acc);
      tc::mma_tf32_ts(d, a + lo + 8 * s, b + (uint64_t)(16 * s), idesc, 1u);
      tc::mma_tf32_ts(d, a + 8 * s, b + blo + (uint64_t)(16 * s), idesc, 1u);
    } else {
      tc::mma_f16_ts(d, a + 8 * s, b + (uint64_t)(16 * s), idesc, acc);
    }
  }
}

// n K steps: the exact unrolled sequence for the common counts, else a plain
// loop (no branch inside either)
template <typename K>
__device__ __forceinline__ void issue_steps(uint32_t d, uint32_t a, uint32_t lo, uint64_t b,
                                            uint64_t blo, uint32_t idesc, int n, bool acc_first) {
  switch (n) {
    case 1: issue_exact<K, 1>(d, a, lo, b, blo, idesc, acc_first); return;
    case 2: issue_exact<K, 2>(d, a, lo, b, blo, idesc, acc_first); return;
    case 3: issue_exact<K, 3>(d, a, lo, b, blo, idesc, acc_first); return;
    case 4: issue_exact<K, 4>(d, a, lo, b, blo, idesc, acc_first); return;
    case 6: issue_exact<K, 6>(d, a, lo, b, blo, idesc, acc_first); return;
    case 8: issue_exact<K, 8>(d, a, lo, b, blo, idesc, acc_first); return;
    default: break;
  }
  if (n <= 0) return;
  issue_exact<K, 1>(d, a, lo, b, blo, idesc, acc_first);
  for (int s = 1; s < n; ++s) {
    if (K::tf32) {
      tc::mma_tf32_ts(d, a + 8 * s, b + (uint64_t)(16 * s), idesc, 1u);
      tc::mma_tf32_ts(d, a + lo + 8 * s, b + (uint64_t)(16 * s), idesc, 1u);
      tc::mma_tf32_ts(d, a + 8 * s, b + blo + (uint64_t)(16 * s), idesc, 1u);
    } else {
      tc::mma_f16_ts(d, a + 8 * s, b + (uint64_t)(16 * s), idesc, 1u);
    }
  }
}

template <typename T, bool HAS_X, int CX, bool IMG>
__global__ void __launch_bounds__(THREADS, 1)
    k_epi_pipe(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmu,
               PipeArgs a, Geom g) {
  using K = PKind<T>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int Ci = a.Ci, Co = a.Co;
  const PipeGeom e = pipe_geom(g, HAS_X, Ci, Co, K::EB, K::tf32, IMG);
  unsigned char *bbase = smem + e.b;
  float2 *twL = reinterpret_cast<float2 *>(smem + e.tw);
  float *bias_s = reinterpret_cast<float *>(smem + e.bias);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + e.bar);
  uint64_t *empty = full + MAX_STAGES;
  uint64_t *aready = empty + MAX_STAGES;
  uint64_t *mdone = aready + 2;
  uint64_t *dempty = mdone + 2;
  uint32_t *tbase_s = reinterpret_cast<uint32_t *>(smem + e.tbase);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NL = g.NL, mL = g.mL;
  const long long SN = (long long)g.S * NL;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, e.cols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      // IMG: the MMAs read the stage itself, so the epilogue warps free it
      // once a tile's MMAs are complete; else the staging warps after copying
      tc::mbar_init(&empty[s], IMG ? NEPI : NCONV);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aready[i], NCONV);
      tc::mbar_init(&mdone[i], 1);
      tc::mbar_init(&dempty[i], NEPI);
    }
    tma::fence_barrier_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    if (HAS_X) tma::prefetch_map(&tmx);
    if (!IMG) tma::prefetch_map(&tmu);
  }
  build_twiddles(twL, NL);
  for (size_t i = (size_t)tid * 16; i < e.NB * e.bbuf; i += THREADS * 16)
    *reinterpret_cast<uint4 *>(bbase + i) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (HAS_X) {  // W in columns [KSp, KSp + Ci) of every B buffer (IMG: [0, Ci)); bias
    const T *W = reinterpret_cast<const T *>(a.W);
    for (int i = tid; i < Co * Ci; i += THREADS) {
      const int o = i / Ci, c = i - o * Ci;
      const float w = to_f<T>(W[i]);
      const uint32_t off = boff(o, (IMG ? 0 : e.KSp) + c, K::EB, e.sbo);
      for (int nb = 0; nb < e.NB; ++nb) bstore1<T>(bbase + nb * e.bbuf, e.bhalf, off, w);
    }
  }
  {
    const T *bias = reinterpret_cast<const T *>(a.bias);
    for (int o = tid; o < 64; o += THREADS)
      bias_s[o] = (HAS_X && bias && o < Co) ? to_f<T>(bias[o]) : 0.f;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;

  const int tps = (int)(SN / ROWS);              // tiles per slab
  const long long ntiles = g.B * g.O * tps;
  const long long per_cta = (ntiles + gridDim.x - 1) / gridDim.x;
  const long long t_begin = blockIdx.x * per_cta;
  const long long t_end = t_begin + per_cta < ntiles ? t_begin + per_cta : ntiles;
  const int ntl = t_begin < t_end ? (int)(t_end - t_begin) : 0;

  if (warp == WARP_TMA) {
    // ---------------------------------------------------------- TMA producer
    // (the whole warp walks the loop and waits; lane 0 issues)
    {
      Cursor c = cursor_at(t_begin, tps, g);
      int j = 0;
      for (; j < ntl; ++j) {
        const int s = j % e.NS;
        const bool ok = j < e.NS || tc::mbar_wait(&empty[s], ((j / e.NS) - 1) & 1, a.err);
        if (!__all_sync(0xffffffffu, ok)) break;     // warp-uniform exit
        if (lane == 0) {
          tma::arrive_expect_tx(&full[s], e.x_bytes + e.u_bytes);
          unsigned char *st = smem + (size_t)s * e.stage;
          if (HAS_X)
            tma::load_4d(st, &tmx, &full[s], c.row0 * NL + c.n0, c.outer, 0, (int)c.b);
          if (IMG)
            tma::load_bulk(st + e.uoff,
                           a.img + ((c.b * g.O + c.outer) * g.S + c.row0) * (size_t)e.u_bytes,
                           e.u_bytes, &full[s]);
          else
            tma::load_4d(st + e.uoff, &tmu, &full[s], c.row0 * 2 * mL, c.outer, 0, (int)c.b);
        }
        __syncwarp();
        cursor_next(c, e.Rt, g);
      }
      // every issued load lands before the CTA may exit
      for (int jj = j - 1; jj >= 0 && jj >= j - e.NS; --jj)
        tc::mbar_wait(&full[jj % e.NS], (jj / e.NS) & 1, nullptr);
    }
  } else if (warp == WARP_MMA) {
    // ---------------------------------------------------------- MMA issuer
    // (the whole warp walks the loop and waits; lane 0 issues)
    {
      Cursor c = cursor_at(t_begin, tps, g);
      const uint32_t idesc = tc::instr_desc(K::fmt, ROWS, e.DA);
      // descriptor offset (16-byte units) of the lo rows of B: after the NP hi rows
      const uint64_t blo_img = K::tf32 ? (uint64_t)(e.NP / 8) * e.sbo_s / 16 : 0;
      const uint64_t blo_buf = K::tf32 ? (uint64_t)(e.bhalf / 16) : 0;
      const uint32_t lo_spec = K::tf32 ? (uint32_t)e.KSp : 0u;
      const uint32_t lo_x = K::tf32 ? (uint32_t)e.KXp : 0u;
      const int ns = e.KSp / K::KSTEP, nx = e.KXp / K::KSTEP;
      // B descriptors of both buffers; one K step advances the start address by
      // 256 bytes (16 in descriptor units, no carry out of the 14-bit field)
      const uint64_t bdesc0 = tc::smem_desc_kmajor(tc::smem_u32(bbase), 128, e.sbo);
      const uint64_t bdesc1 =
          tc::smem_desc_kmajor(tc::smem_u32(bbase + (e.NB - 1) * e.bbuf), 128, e.sbo);
      int j = 0;
      for (; j < ntl; ++j) {
        bool ok = tc::mbar_wait(&aready[j & 1], (j >> 1) & 1, a.err);
        if (ok && j >= 2) ok = tc::mbar_wait(&dempty[j & 1], ((j - 2) >> 1) & 1, a.err);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc::fence_after_sync();
        const int variant = e.Rt > 1 ? 0 : c.n0 / ROWS;
        const int ab = e.NA == 2 ? (j & 1) : 0;
        const uint32_t d = tbase + (uint32_t)((j & 1) * e.DA);
        // one elected thread issues the tile's K steps (tf32: A_hi B_hi, A_lo B_hi
        // and A_hi B_lo of each K step into one accumulator of NP columns, so the
        // epilogue reads one column set); one K step advances B by 256 bytes (16
        // in descriptor units, no carry out of the 14-bit field) and A by 8 TMEM
        // columns
        if (tc::elect_one()) {
          // IMG: the spectral steps read this tile's ring stage, the x steps W;
          // else both read the staged B buffer, the x steps after the spectral
          const uint64_t bspec =
              IMG ? tc::smem_desc_kmajor(
                        tc::smem_u32(smem + (size_t)(j % e.NS) * e.stage + e.uoff), 128, e.sbo_s)
                  : (ab ? bdesc1 : bdesc0);
          const uint64_t bx = IMG ? bdesc0 : bspec + (uint64_t)(16 * ns);
          issue_steps<K>(d, tbase + e.col_spec + variant * e.cs_cols, lo_spec, bspec,
                         IMG ? blo_img : blo_buf, idesc, ns, false);
          issue_steps<K>(d, tbase + e.col_x + ab * e.ax_cols, lo_x, bx, blo_buf, idesc, nx, true);
          tc::mma_commit(&mdone[j & 1]);
        }
        __syncwarp();
        cursor_next(c, e.Rt, g);
      }
      // no MMA may still run when TMEM is freed
      if (j > 0) tc::mbar_wait(&mdone[(j - 1) & 1], ((j - 1) >> 1) & 1, nullptr);
    }
  } else if (warp < NCONV) {
    // ---------------------------------------------------------- staging
    // two warps per TMEM lane quarter: point t, and half `shalf` of the x
    // channel groups and of the B chunks
    const int t = tid & (ROWS - 1);                     // point / TMEM lane
    const int shalf = tid / ROWS;
    const uint32_t arow = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t lo_spec = K::tf32 ? (uint32_t)e.KSp : 0u;
    const uint32_t lo_x = K::tf32 ? (uint32_t)e.KXp : 0u;
    // resident spectral A block per variant: row t = point n0 + t (NL >= 128)
    // or point t of the Rt rows (NL < 128): (cos, -sin)(2 pi k n / NL) in the
    // slot of the point's row, zeros elsewhere
    for (int v = 0; v < (shalf == 0 ? e.nvar : 0); ++v) {
      const int n = e.Rt > 1 ? t % NL : v * ROWS + t;
      const int rl = e.Rt > 1 ? t / NL : 0;
      const uint32_t c0v = arow + e.col_spec + v * e.cs_cols;
      int r = 0, k = 0, par = 0, idx = 0;
      for (int c0 = 0; c0 < e.KSp; c0 += 16) {
        float vals[16];
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
        stage16<T>(c0v + (K::tf32 ? c0 : c0 / 2), lo_spec, vals);
      }
    }
    const int njb = e.KS / 4;                           // 16-byte chunks per U row
    const int nchunk = rup(Co, 8) * njb;
    const int two_ml = 2 * mL;
    // This thread's chunks of the B spectral block are the same for every
    // tile: chunk i = tid + 256 m.  Chunk order walks 8-row groups diagonally so a
    // quarter warp touches 8 distinct 16-byte bank groups on both the read and
    // the write side.  Packed per slot: source float index (low 16 bits), B byte
    // offset (high 16 bits); bias_mask bit m: add the bias (k = 0 real column).
    constexpr int MAXSLOT = 4;
    constexpr int NSTG = NCONV * 32;
    uint32_t slot[MAXSLOT];
    float slot_bias[MAXSLOT];
    const bool slots_fit = nchunk <= MAXSLOT * NSTG && e.bhalf <= 65536;
#pragma unroll
    for (int m = 0; m < MAXSLOT; ++m) {
      slot[m] = 0xffffffffu;
      slot_bias[m] = 0.f;
      const int i = tid + NSTG * m;
      if (slots_fit && i < nchunk) {
        const int o8 = i / (8 * njb), rem = i - o8 * 8 * njb;
        const int ol = rem & 7, jrot = rem >> 3;
        const int jb = (jrot + ol) % njb;
        const int o = o8 * 8 + ol;
        if (o < Co) {
          slot[m] = (uint32_t)(o * e.KS + 4 * jb) | (boff(o, 4 * jb, K::EB, e.sbo) << 16);
          if (HAS_X && (4 * jb) % two_ml == 0) slot_bias[m] = bias_s[o];
        }
      }
    }
    for (int j = 0; j < ntl; ++j) {
      const int s = j % e.NS;
      const int ab = e.NA == 2 ? (j & 1) : 0;
      bool ok = tc::mbar_wait(&full[s], (j / e.NS) & 1, a.err);
      if (ok && j >= e.NA)
        ok = tc::mbar_wait(&mdone[(j - e.NA) & 1], ((j - e.NA) >> 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, ok)) break;      // warp-uniform exit
      tc::fence_after_sync();
      const unsigned char *st = smem + (size_t)s * e.stage;
      // B spectral block: U rows -> K-major core matrices (IMG: prebuilt)
      if (IMG) {
      } else if (slots_fit) {
        const float *us = reinterpret_cast<const float *>(st + e.uoff);
        unsigned char *bh = bbase + ab * e.bbuf;
        float4 v[MAXSLOT];
#pragma unroll
        for (int m = 0; m < MAXSLOT; ++m)
          if (slot[m] != 0xffffffffu)
            v[m] = *reinterpret_cast<const float4 *>(us + (slot[m] & 0xffffu));
#pragma unroll
        for (int m = 0; m < MAXSLOT; ++m) {
          if (slot[m] != 0xffffffffu) {
            v[m].x += slot_bias[m];
            bstore4<T>(bh, e.bhalf, slot[m] >> 16, v[m]);
          }
        }
      } else {
        const float *us = reinterpret_cast<const float *>(st + e.uoff);
        unsigned char *bh = bbase + ab * e.bbuf;
        for (int i = tid; i < nchunk; i += NSTG) {
          const int o8 = i / (8 * njb), rem = i - o8 * 8 * njb;
          const int ol = rem & 7, jrot = rem >> 3;
          const int jb = (jrot + ol) % njb;
          const int o = o8 * 8 + ol;
          if (o < Co) {
            float4 v = *reinterpret_cast<const float4 *>(us + o * e.KS + 4 * jb);
            if (HAS_X && (4 * jb) % two_ml == 0) v.x += bias_s[o];
            bstore4<T>(bh, e.bhalf, boff(o, 4 * jb, K::EB, e.sbo), v);
          }
        }
      }
      if (HAS_X) {
        const T *xs = reinterpret_cast<const T *>(st);
        const uint32_t xc = arow + e.col_x + ab * e.ax_cols;
#pragma unroll
        for (int c0 = 0; c0 < CX; c0 += 16) {
          if (c0 < e.KXp && ((c0 >> 4) & 1) == shalf) {
            float vals[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              vals[i] = c0 + i < Ci ? to_f<T>(xs[(c0 + i) * ROWS + t]) : 0.f;
            stage16<T>(xc + (K::tf32 ? c0 : c0 / 2), lo_x, vals);
          }
        }
      }
      __syncwarp();
      if (!IMG && lane == 0) tma::arrive(&empty[s]);    // the stage may be refilled
      tc::tmem_wait_st();
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(&aready[j & 1]);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3, half = (warp - NCONV) >> 2;
    const int t = q * 32 + lane;
    const uint32_t arow = tbase + ((uint32_t)(q * 32) << 16);
    const long long cstride = (long long)g.O * SN;
    T *out = reinterpret_cast<T *>(a.out);
    T *pre_out = reinterpret_cast<T *>(a.pre_out);
    constexpr int GPH = CX / 32 > 0 ? CX / 32 : 1;     // channel groups (of 16) per half
    Cursor c = cursor_at(t_begin, tps, g);
    for (int j = 0; j < ntl; ++j) {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&mdone[j & 1], (j >> 1) & 1, a.err))) break;
      tc::fence_after_sync();
      if (IMG && lane == 0) tma::arrive(&empty[j % e.NS]);   // tile j's MMAs are done with it
      const uint32_t dcol = arow + (uint32_t)((j & 1) * e.DA);
      float v[GPH][16];
#pragma unroll
      for (int gi = 0; gi < GPH; ++gi) {
        const int c0 = (2 * gi + half) * 16;
        if (c0 < Co) {
          uint32_t dv[16];
          tc::tmem_ld16(dcol + c0, dv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[gi][i] = __uint_as_float(dv[i]);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(&dempty[j & 1]);       // D buffer may be overwritten
      const long long ob =
          (c.b * Co * g.O + c.outer) * SN + (long long)c.row0 * NL + c.n0 + t;
#pragma unroll
      for (int gi = 0; gi < GPH; ++gi) {
        const int c0 = (2 * gi + half) * 16;
        if (c0 < Co) {
          const int nv = Co - c0 < 16 ? Co - c0 : 16;
          if (HAS_X && pre_out) {
            T *pp = pre_out + ob + (long long)c0 * cstride;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (i < nv) *pp = from_f<T>(v[gi][i]);
              pp += cstride;
            }
          }
          if (HAS_X && a.act) {
#pragma unroll
            for (int i = 0; i < 16; i += 2) gelu2(v[gi][i], v[gi][i + 1]);
          }
          T *op = out + ob + (long long)c0 * cstride;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (i < nv) *op = from_f<T>(v[gi][i]);
            op += cstride;
          }
        }
      }
      cursor_next(c, e.Rt, g);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, e.cols);
  }
}

template <typename T, bool HAS_X, bool IMG>
cudaError_t launch_pipe_t(const Launch &L, const Geom &g, const PipeArgs &a, const void *x,
                          const float2 *U) {
  using K = PKind<T>;
  const PipeGeom e = pipe_geom(g, HAS_X, a.Ci, a.Co, K::EB, K::tf32, IMG);
  const long long SN = (long long)g.S * g.NL;
  CUtensorMap tmx, tmu;
  memset(&tmx, 0, sizeof(tmx));
  memset(&tmu, 0, sizeof(tmu));
  if (HAS_X) {
    const uint64_t dims[4] = {(uint64_t)SN, (uint64_t)g.O, (uint64_t)a.Ci, (uint64_t)g.B};
    const uint64_t str[3] = {(uint64_t)SN * K::EB, (uint64_t)g.O * SN * K::EB,
                             (uint64_t)a.Ci * g.O * SN * K::EB};
    const uint32_t box[4] = {(uint32_t)ROWS, 1u, (uint32_t)a.Ci, 1u};
    if (!encode_tmap_4d(&tmx, K::tmap, x, dims, str, box)) return cudaErrorInvalidValue;
  }
  if (!IMG) {
    const uint64_t row = (uint64_t)g.S * 2 * g.mL;   // floats of one (b, o, outer) slab
    const uint64_t dims[4] = {row, (uint64_t)g.O, (uint64_t)a.Co, (uint64_t)g.B};
    const uint64_t str[3] = {row * 4, (uint64_t)g.O * row * 4, (uint64_t)a.Co * g.O * row * 4};
    const uint32_t box[4] = {(uint32_t)e.KS, 1u, (uint32_t)a.Co, 1u};
    if (!encode_tmap_4d(&tmu, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, U, dims, str, box))
      return cudaErrorInvalidValue;
  }
  const long long ntiles = g.B * g.O * (SN / ROWS);
  const int grid = (int)(ntiles < L.num_sms ? ntiles : L.num_sms);
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)e.total);
    kern<<<grid, THREADS, e.total, L.stream>>>(tmx, tmu, a, g);
  };
  const int cmax = a.Co > a.Ci ? a.Co : a.Ci;
  if (cmax <= 16) go(k_epi_pipe<T, HAS_X, 16, IMG>);
  else if (cmax <= 32) go(k_epi_pipe<T, HAS_X, 32, IMG>);
  else go(k_epi_pipe<T, HAS_X, 64, IMG>);
  return cudaGetLastError();
}

template <typename T, bool HAS_X>
cudaError_t launch_pipe_img(const Launch &L, const Geom &g, const PipeArgs &a, const void *x,
                            const float2 *U) {
  return a.img ? launch_pipe_t<T, HAS_X, true>(L, g, a, x, U)
               : launch_pipe_t<T, HAS_X, false>(L, g, a, x, U);
}

// ===========================================================================
// Block backward (step S6, 16-bit storage) as a warp-specialised tcgen05
// pipeline.  For a tile of 128 consecutive grid points p:
//     dz[p, o] = dy[p, o] GELU'(pre[p, o])
//     dx[p, i] = sum_j basis[p, j] Udx[i, j] + sum_o dz[p, o] W[o, i]
//     dW[o, i] += sum_p dz[p, o] x[p, i],  db[o] += sum_p dz[p, o]
// Udx is the spectrum of dxhat inverted along the slab axis (the slab-axis
// inverse kernel), basis the last-axis inverse basis of the forward.  The dx
// chain is the forward epilogue's GEMM with dz in place of x and W^T in place
// of W; the dW chain reads the x tile straight from the ring stage (TMA with
// 128-byte swizzle, the K-major layout the tensor core reads) against dz^T,
// which the staging warps write to shared memory, and accumulates in a TMEM
// accumulator that persists over all tiles of the CTA.  Sixteen rows of ones
// after the x rows make the last sixteen accumulator columns db.
//
//   warp 25       TMA producer: x (two 64-point boxes, swizzled), dy, pre and
//                 the Udx rows of tile j into ring stage j % NS
//   warps 0-15    staging, four per TMEM lane quarter, one 16-channel group
//                 each: dz -> A (TMEM) and dz^T -> A_dW (shared memory); Udx
//                 rows -> the spectral columns of the dx B operand
//   warp 24       MMA issuer: both chains of tile j; one commit frees the ring
//                 stage, another signals D_dx full and the A/B buffers free
//   warps 16-23   epilogue: D_dx -> dx; at the end, D_dW -> per-CTA partials
// ===========================================================================
constexpr int BW_NCONV = 16, BW_NEPI = 8;
constexpr int BW_WARP_MMA = BW_NCONV + BW_NEPI;   // 24
constexpr int BW_WARP_TMA = BW_WARP_MMA + 1;      // 25
constexpr int BW_THREADS = (BW_WARP_TMA + 1) * 32;
constexpr int BW_MAX_STAGES = 4;
constexpr int BW_XBOX = 64;                       // points per swizzled x box (128 bytes)

struct BwdGeom {
  int Rt, nvar, KS, KSp, KA, NW, NS, NAW;
  int col_dw, col_spec, col_z, used_cols, cols, cs_cols;
  uint32_t sbo, sbo_w, bytes_tx;
  size_t xbox, x_off, dy_off, pre_off, u_off, stage, bbuf, abuf, b, aw, tw, bar, tbase, total;
};

// 16-bit storage only (eb = 2); requires Ci % 16 == 0 and Co % 16 == 0
__host__ __device__ inline BwdGeom bwd_geom(const Geom &g, int Ci, int Co, bool act) {
  BwdGeom e;
  e.Rt = g.NL >= ROWS ? 1 : ROWS / g.NL;
  e.nvar = g.NL >= ROWS ? g.NL / ROWS : 1;
  e.KS = e.Rt * 2 * g.mL;
  e.KSp = rup(e.KS, 16);
  e.KA = e.KSp + Co;                       // K of the dx chain: spectral, then dz
  e.NW = Ci + 16;                          // N of the dW chain: x rows, then ones
  e.cs_cols = e.KSp / 2;
  e.col_dw = 2 * Ci;                       // two D_dx buffers first
  e.col_spec = e.col_dw + rup(e.NW, 16);
  e.col_z = e.col_spec + e.nvar * e.cs_cols;
  e.used_cols = e.col_z + 2 * (Co / 2);
  e.cols = 32;
  while (e.cols < e.used_cols && e.cols < 1024) e.cols *= 2;
  e.sbo = (uint32_t)(e.KA * 2 / 16) * 128u;
  e.sbo_w = (uint32_t)(ROWS * 2 / 16) * 128u;
  e.xbox = (size_t)e.NW * 128;             // one swizzled box: NW rows of 128 bytes
  e.x_off = 0;
  e.dy_off = alg(e.x_off + 2 * e.xbox, 1024);
  e.pre_off = alg(e.dy_off + (size_t)Co * ROWS * 2, 128);
  e.u_off = alg(e.pre_off + (act ? (size_t)Co * ROWS * 2 : 0), 128);
  e.stage = alg(e.u_off + (size_t)Ci * e.KS * 4, 1024);
  e.bytes_tx = (uint32_t)(2 * (size_t)Ci * 128 + (size_t)Co * ROWS * 2 * (act ? 2 : 1) +
                          (size_t)Ci * e.KS * 4);
  e.bbuf = alg((size_t)Ci * e.KA * 2, 1024);
  e.abuf = (size_t)ROWS * ROWS * 2;        // dz^T: 128 rows (o, zero past Co) x 128 points
  const size_t fixed_base = 2 * e.bbuf + alg(sizeof(float2) * g.NL, 128) +
                            sizeof(uint64_t) * (2 * BW_MAX_STAGES + 6) + 16;
  size_t room2 = 232448 > fixed_base + 2 * e.abuf ? 232448 - fixed_base - 2 * e.abuf : 0;
  e.NAW = room2 / e.stage >= 2 ? 2 : 1;
  const size_t room = 232448 > fixed_base + e.NAW * e.abuf ? 232448 - fixed_base - e.NAW * e.abuf : 0;
  const size_t ns = room / e.stage;
  e.NS = (int)(ns < (size_t)BW_MAX_STAGES ? ns : (size_t)BW_MAX_STAGES);
  size_t off = (size_t)(e.NS > 0 ? e.NS : 0) * e.stage;
  e.b = off; off += 2 * e.bbuf;
  e.aw = off; off += e.NAW * e.abuf;
  e.tw = off; off = alg(off + sizeof(float2) * g.NL, 128);
  e.bar = off; off += sizeof(uint64_t) * (2 * BW_MAX_STAGES + 6);
  e.tbase = off; off += 16;
  e.total = off < 116 * 1024 ? 116 * 1024 : off;
  return e;
}

// K-major, 128-byte swizzle descriptor (8-row groups 1024 bytes apart): the
// layout a TMA box with a 128-byte inner extent and 128-byte swizzle writes
__device__ __forceinline__ uint64_t desc_sw128_b(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// the dW chain of one tile: 8 K steps of 16 points; A = dz^T (no swizzle,
// 256 bytes per step), B = the x boxes (32 bytes per step inside a 128-byte
// swizzle atom, four steps per box)
__device__ __forceinline__ void issue_dw(uint32_t d, uint64_t adesc, uint64_t xdesc0,
                                         uint64_t xdesc1, uint32_t idesc, bool acc_first) {
#pragma unroll
  for (int s = 0; s < ROWS / 16; ++s) {
    const uint64_t bd = (s < 4 ? xdesc0 : xdesc1) + (uint64_t)(2 * (s & 3));
    tc::mma_f16_ss(d, adesc + (uint64_t)(16 * s), bd, idesc, (acc_first || s > 0) ? 1u : 0u);
  }
}

template <typename T, int CX>
__global__ void __launch_bounds__(BW_THREADS, 1)
    k_epi_bwd_pipe(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmdy,
                   const __grid_constant__ CUtensorMap tmpre,
                   const __grid_constant__ CUtensorMap tmu, PipeArgs a, float *partial, Geom g) {
  using K = PKind<T>;
  static_assert(!PKind<T>::tf32, "16-bit storage only");
  extern __shared__ __align__(1024) unsigned char smem[];
  const int Ci = a.Ci, Co = a.Co;
  const bool act = a.act != 0;
  const BwdGeom e = bwd_geom(g, Ci, Co, act);
  unsigned char *bbase = smem + e.b;
  unsigned char *awbase = smem + e.aw;
  float2 *twL = reinterpret_cast<float2 *>(smem + e.tw);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + e.bar);
  uint64_t *empty = full + BW_MAX_STAGES;
  uint64_t *aready = empty + BW_MAX_STAGES;
  uint64_t *mdone = aready + 2;
  uint64_t *dempty = mdone + 2;
  uint32_t *tbase_s = reinterpret_cast<uint32_t *>(smem + e.tbase);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NL = g.NL, mL = g.mL;
  const long long SN = (long long)g.S * NL;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, e.cols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < BW_MAX_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);       // the tile's MMA commit
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aready[i], BW_NCONV);
      tc::mbar_init(&mdone[i], 1);
      tc::mbar_init(&dempty[i], BW_NEPI);
    }
    tma::fence_barrier_init();
  }
  if (warp == BW_WARP_TMA && lane == 0) {
    tma::prefetch_map(&tmx);
    tma::prefetch_map(&tmdy);
    if (act) tma::prefetch_map(&tmpre);
    tma::prefetch_map(&tmu);
  }
  build_twiddles(twL, NL);
  // zero the B buffers and the dz^T buffers (rows past Co stay zero); the ones
  // rows after the x rows of every box of every stage (any swizzle of ones is
  // ones)
  for (size_t i = (size_t)tid * 16; i < 2 * e.bbuf + e.NAW * e.abuf; i += BW_THREADS * 16)
    *reinterpret_cast<uint4 *>(bbase + i) = make_uint4(0, 0, 0, 0);
  {
    const uint32_t one2 = PKind<T>::fmt == tc::FMT_BF16 ? 0x3F803F80u : 0x3C003C00u;
    const int per_box = 16 * 128 / 16;      // 16-byte chunks of the ones rows of one box
    for (int i = tid; i < e.NS * 2 * per_box; i += BW_THREADS) {
      const int sb = i / per_box, c = i - sb * per_box;
      unsigned char *dst = smem + (size_t)(sb >> 1) * e.stage + e.x_off + (size_t)(sb & 1) * e.xbox +
                           (size_t)Ci * 128 + (size_t)c * 16;
      *reinterpret_cast<uint4 *>(dst) = make_uint4(one2, one2, one2, one2);
    }
  }
  __syncthreads();
  {  // W^T in columns [KSp, KSp + Co) of both B buffers: B[n = i][k = KSp + o] = W[o][i]
    const T *W = reinterpret_cast<const T *>(a.W);
    for (int idx = tid; idx < Co * Ci; idx += BW_THREADS) {
      const int o = idx / Ci, i = idx - o * Ci;
      const uint32_t off = boff(i, e.KSp + o, 2, e.sbo);
      for (int nb = 0; nb < 2; ++nb) *reinterpret_cast<T *>(bbase + nb * e.bbuf + off) = W[idx];
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;

  const int tps = (int)(SN / ROWS);
  const long long ntiles = g.B * g.O * tps;
  const long long per_cta = (ntiles + gridDim.x - 1) / gridDim.x;
  const long long t_begin = blockIdx.x * per_cta;
  const long long t_end = t_begin + per_cta < ntiles ? t_begin + per_cta : ntiles;
  const int ntl = t_begin < t_end ? (int)(t_end - t_begin) : 0;

  if (warp == BW_WARP_TMA) {
    // ---------------------------------------------------------- TMA producer
    Cursor c = cursor_at(t_begin, tps, g);
    int j = 0;
    for (; j < ntl; ++j) {
      const int s = j % e.NS;
      const bool ok = j < e.NS || tc::mbar_wait(&empty[s], ((j / e.NS) - 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (lane == 0) {
        unsigned char *st = smem + (size_t)s * e.stage;
        const int p0 = c.row0 * NL + c.n0;
        tma::arrive_expect_tx(&full[s], e.bytes_tx);
        tma::load_4d(st + e.x_off, &tmx, &full[s], p0, c.outer, 0, (int)c.b);
        tma::load_4d(st + e.x_off + e.xbox, &tmx, &full[s], p0 + BW_XBOX, c.outer, 0, (int)c.b);
        tma::load_4d(st + e.dy_off, &tmdy, &full[s], p0, c.outer, 0, (int)c.b);
        if (act) tma::load_4d(st + e.pre_off, &tmpre, &full[s], p0, c.outer, 0, (int)c.b);
        tma::load_4d(st + e.u_off, &tmu, &full[s], c.row0 * 2 * mL, c.outer, 0, (int)c.b);
      }
      __syncwarp();
      cursor_next(c, e.Rt, g);
    }
    for (int jj = j - 1; jj >= 0 && jj >= j - e.NS; --jj)
      tc::mbar_wait(&full[jj % e.NS], (jj / e.NS) & 1, nullptr);
  } else if (warp == BW_WARP_MMA) {
    // ---------------------------------------------------------- MMA issuer
    Cursor c = cursor_at(t_begin, tps, g);
    const uint32_t idx_desc = tc::instr_desc(K::fmt, ROWS, Ci);
    const uint32_t idw_desc = tc::instr_desc(K::fmt, ROWS, e.NW);
    const int nss = e.KSp / 16, nzs = Co / 16;
    int j = 0;
    for (; j < ntl; ++j) {
      bool ok = tc::mbar_wait(&aready[j & 1], (j >> 1) & 1, a.err);
      if (ok && j >= 2) ok = tc::mbar_wait(&dempty[j & 1], ((j - 2) >> 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::fence_after_sync();
      const int s = j % e.NS;
      const int variant = e.Rt > 1 ? 0 : c.n0 / ROWS;
      if (tc::elect_one()) {
        const uint32_t d = tbase + (uint32_t)((j & 1) * Ci);
        const uint64_t bdesc =
            tc::smem_desc_kmajor(tc::smem_u32(bbase + (j & 1) * e.bbuf), 128, e.sbo);
        // dx: spectral steps (resident basis A, Udx columns of B), then dz steps
        issue_steps<K>(d, tbase + e.col_spec + variant * e.cs_cols, 0u, bdesc, 0u, idx_desc,
                       nss, false);
        issue_steps<K>(d, tbase + e.col_z + (j & 1) * (Co / 2), 0u,
                       bdesc + (uint64_t)(16 * nss), 0u, idx_desc, nzs, true);
        // dW, db: A = dz^T, B = the stage's x boxes and ones rows
        const unsigned char *xs = smem + (size_t)s * e.stage + e.x_off;
        issue_dw(tbase + e.col_dw,
                 tc::smem_desc_kmajor(tc::smem_u32(awbase + (j % e.NAW) * e.abuf), 128, e.sbo_w),
                 desc_sw128_b(tc::smem_u32(xs)), desc_sw128_b(tc::smem_u32(xs + e.xbox)),
                 idw_desc, j > 0);
        tc::mma_commit(&empty[s]);
        tc::mma_commit(&mdone[j & 1]);
      }
      __syncwarp();
      cursor_next(c, e.Rt, g);
    }
    if (j > 0) tc::mbar_wait(&mdone[(j - 1) & 1], ((j - 1) >> 1) & 1, nullptr);
  } else if (warp < BW_NCONV) {
    // ---------------------------------------------------------- staging
    const int t = tid & (ROWS - 1);
    const int part = tid / ROWS;               // 16-channel groups part, part + 4, ..
    const uint32_t arow = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    // resident spectral A per variant, as in the forward (16-bit: two per column)
    for (int v = 0; v < (part == 0 ? e.nvar : 0); ++v) {
      const int n = e.Rt > 1 ? t % NL : v * ROWS + t;
      const int rl = e.Rt > 1 ? t / NL : 0;
      const uint32_t c0v = arow + e.col_spec + v * e.cs_cols;
      int r = 0, k = 0, par = 0, idx = 0;
      for (int c0 = 0; c0 < e.KSp; c0 += 16) {
        float vals[16];
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
        stage16<T>(c0v + c0 / 2, 0u, vals);
      }
    }
    const int njb = e.KS / 4;                 // 16-byte chunks of one Udx row
    const int nchunk = Ci * njb;
    constexpr int NSTG = BW_NCONV * 32;
    for (int j = 0; j < ntl; ++j) {
      const int s = j % e.NS;
      const int ab = j & 1, aw = j % e.NAW;
      bool ok = tc::mbar_wait(&full[s], (j / e.NS) & 1, a.err);
      // A_dz / B buffer ab were last read by tile j - 2; dz^T buffer aw by tile j - NAW
      if (ok && j >= 2) ok = tc::mbar_wait(&mdone[ab], ((j - 2) >> 1) & 1, a.err);
      if (ok && e.NAW == 1 && j >= 1)
        ok = tc::mbar_wait(&mdone[(j - 1) & 1], ((j - 1) >> 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc::fence_after_sync();
      const unsigned char *st = smem + (size_t)s * e.stage;
      // Udx rows -> B[n = i][k < KS], chunks of four K values
      {
        const float *us = reinterpret_cast<const float *>(st + e.u_off);
        unsigned char *bh = bbase + ab * e.bbuf;
        for (int i = tid; i < nchunk; i += NSTG) {
          const int o8 = i / (8 * njb), rem = i - o8 * 8 * njb;
          const int ol = rem & 7, jrot = rem >> 3;
          const int jb = (jrot + ol) % njb;
          const int ch = o8 * 8 + ol;
          const float4 v = *reinterpret_cast<const float4 *>(us + ch * e.KS + 4 * jb);
          bstore4<T>(bh, 0, boff(ch, 4 * jb, 2, e.sbo), v);
        }
      }
      // dz = dy GELU'(pre): this half's 16-channel groups -> A (TMEM) and dz^T
      {
        const T *dys = reinterpret_cast<const T *>(st + e.dy_off);
        const T *prs = reinterpret_cast<const T *>(st + e.pre_off);
        const uint32_t zc = arow + e.col_z + ab * (Co / 2);
        unsigned char *awb = awbase + aw * e.abuf;
#pragma unroll
        for (int c0 = 0; c0 < CX; c0 += 16) {
          if (c0 < Co && ((c0 >> 4) & 3) == part) {
            float vals[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) vals[i] = to_f<T>(dys[(c0 + i) * ROWS + t]);
            if (act) {
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                float g0 = to_f<T>(prs[(c0 + i) * ROWS + t]);
                float g1 = to_f<T>(prs[(c0 + i + 1) * ROWS + t]);
                gelu_grad2(g0, g1);
                vals[i] *= g0;
                vals[i + 1] *= g1;
              }
            }
            stage16<T>(zc + c0 / 2, 0u, vals);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              *reinterpret_cast<T *>(awb + boff(c0 + i, t, 2, e.sbo_w)) = from_f<T>(vals[i]);
          }
        }
      }
      tc::tmem_wait_st();
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(&aready[ab]);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3, half = (warp - BW_NCONV) >> 2;
    const int t = q * 32 + lane;
    const uint32_t arow = tbase + ((uint32_t)(q * 32) << 16);
    const long long cstride = (long long)g.O * SN;
    T *out = reinterpret_cast<T *>(a.out);
    Cursor c = cursor_at(t_begin, tps, g);
    int j = 0;
    for (; j < ntl; ++j) {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&mdone[j & 1], (j >> 1) & 1, a.err))) break;
      tc::fence_after_sync();
      const uint32_t dcol = arow + (uint32_t)((j & 1) * Ci);
      constexpr int GPH = CX / 32 > 0 ? CX / 32 : 1;
      float v[GPH][16];
#pragma unroll
      for (int gi = 0; gi < GPH; ++gi) {
        const int c0 = (2 * gi + half) * 16;
        if (c0 < Ci) {
          uint32_t dv[16];
          tc::tmem_ld16(dcol + c0, dv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[gi][i] = __uint_as_float(dv[i]);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(&dempty[j & 1]);
      const long long ob = (c.b * Ci * g.O + c.outer) * SN + (long long)c.row0 * NL + c.n0 + t;
#pragma unroll
      for (int gi = 0; gi < GPH; ++gi) {
        const int c0 = (2 * gi + half) * 16;
        if (c0 < Ci) {
          T *op = out + ob + (long long)c0 * cstride;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            *op = from_f<T>(v[gi][i]);
            op += cstride;
          }
        }
      }
      cursor_next(c, e.Rt, g);
    }
    // all of the CTA's MMAs are complete once the last tile's mdone has been
    // seen (or there were none): D_dW row o = lane t -> partial[cta][o][0..Ci]
    const bool all_seen = __all_sync(0xffffffffu, j == ntl);
    tc::fence_after_sync();
    float *dst = partial + (long long)blockIdx.x * Co * (Ci + 1);
    const bool row = t < Co;
    for (int c0 = half * 16; c0 < e.NW; c0 += 32) {
      uint32_t dv[16];
      tc::tmem_ld16(arow + e.col_dw + c0, dv);
      tc::tmem_wait_ld();
      if (row && all_seen) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int col = c0 + i;
          const float val = ntl > 0 ? __uint_as_float(dv[i]) : 0.f;
          if (col < Ci) dst[t * (Ci + 1) + col] = val;
          else if (col == Ci) dst[t * (Ci + 1) + Ci] = val;
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, e.cols);
  }
}

template <typename T>
cudaError_t launch_bwd_pipe_t(const Launch &L, const Geom &g, const PipeArgs &a, const void *x,
                              const void *dy, const void *pre, const float2 *U, float *partial,
                              int *nparts) {
  using K = PKind<T>;
  const bool act = a.act != 0;
  const BwdGeom e = bwd_geom(g, a.Ci, a.Co, act);
  const long long SN = (long long)g.S * g.NL;
  CUtensorMap tmx, tmdy, tmpre, tmu;
  memset(&tmx, 0, sizeof(tmx));
  memset(&tmdy, 0, sizeof(tmdy));
  memset(&tmpre, 0, sizeof(tmpre));
  memset(&tmu, 0, sizeof(tmu));
  {
    const uint64_t dims[4] = {(uint64_t)SN, (uint64_t)g.O, (uint64_t)a.Ci, (uint64_t)g.B};
    const uint64_t str[3] = {(uint64_t)SN * 2, (uint64_t)g.O * SN * 2,
                             (uint64_t)a.Ci * g.O * SN * 2};
    const uint32_t box[4] = {(uint32_t)BW_XBOX, 1u, (uint32_t)a.Ci, 1u};
    if (!encode_tmap_4d(&tmx, K::tmap, x, dims, str, box, true)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[4] = {(uint64_t)SN, (uint64_t)g.O, (uint64_t)a.Co, (uint64_t)g.B};
    const uint64_t str[3] = {(uint64_t)SN * 2, (uint64_t)g.O * SN * 2,
                             (uint64_t)a.Co * g.O * SN * 2};
    const uint32_t box[4] = {(uint32_t)ROWS, 1u, (uint32_t)a.Co, 1u};
    if (!encode_tmap_4d(&tmdy, K::tmap, dy, dims, str, box)) return cudaErrorInvalidValue;
    if (act && !encode_tmap_4d(&tmpre, K::tmap, pre, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t row = (uint64_t)g.S * 2 * g.mL;
    const uint64_t dims[4] = {row, (uint64_t)g.O, (uint64_t)a.Ci, (uint64_t)g.B};
    const uint64_t str[3] = {row * 4, (uint64_t)g.O * row * 4, (uint64_t)a.Ci * g.O * row * 4};
    const uint32_t box[4] = {(uint32_t)e.KS, 1u, (uint32_t)a.Ci, 1u};
    if (!encode_tmap_4d(&tmu, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, U, dims, str, box))
      return cudaErrorInvalidValue;
  }
  const long long ntiles = g.B * g.O * (SN / ROWS);
  const int grid = (int)(ntiles < L.num_sms ? ntiles : L.num_sms);
  *nparts = grid;
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)e.total);
    kern<<<grid, BW_THREADS, e.total, L.stream>>>(tmx, tmdy, tmpre, tmu, a, partial, g);
  };
  const int cmax = a.Co > a.Ci ? a.Co : a.Ci;
  if (cmax <= 16) go(k_epi_bwd_pipe<T, 16>);
  else if (cmax <= 32) go(k_epi_bwd_pipe<T, 32>);
  else go(k_epi_bwd_pipe<T, 64>);
  return cudaGetLastError();
}

}  // namespace

bool epi_pipe_supported(const Geom &g, int dtype, int mode, int Ci, int Co, const void *x,
                        const void *U) {
  if (mode != EPI_SPEC && mode != EPI_BLOCK_FWD) return false;
  const bool has_x = mode == EPI_BLOCK_FWD;
  if (!(g.NL % ROWS == 0 || ROWS % g.NL == 0)) return false;
  const long long SN = (long long)g.S * g.NL;
  if (SN % ROWS != 0 || SN > (1LL << 30) || g.B > (1LL << 30)) return false;
  // U rows through TMA: 16-byte aligned row starts and box widths
  if (g.mL % 2 != 0) return false;
  if ((reinterpret_cast<uintptr_t>(U) & 15) != 0) return false;
  if (has_x && (reinterpret_cast<uintptr_t>(x) & 15) != 0) return false;
  const bool tf32 = dtype == DT_F32;
  const PipeGeom e = pipe_geom(g, has_x, Ci, Co, tf32 ? 4 : 2, tf32);
  if (e.KS > 256 || e.DC > 256 || e.used_cols > 512) return false;
  if (e.NS < 2 || e.total > kSmemMax) return false;
  return true;
}

bool epi_img_supported(const Geom &g, int dtype, int mode, int Ci, int Co) {
  if (mode != EPI_SPEC && mode != EPI_BLOCK_FWD) return false;
  if (g.d != 2 || g.NL < ROWS || Co % 16 != 0 || (2 * g.mL) % 16 != 0) return false;
  const bool tf32 = dtype == DT_F32;
  const PipeGeom e = pipe_geom(g, mode == EPI_BLOCK_FWD, Ci, Co, tf32 ? 4 : 2, tf32, true);
  return e.NS >= 2 && e.total <= kSmemMax && e.KS == e.KSp;
}

size_t epi_img_row_bytes(int dtype, int Co, int mL) {
  return (size_t)(dtype == DT_F32 ? 2 * Co : Co) * 2 * mL * (dtype == DT_F32 ? 4 : 2);
}

cudaError_t launch_epi_pipe(const Launch &L, const Geom &g, int dtype, int mode,
                            const EpiArgs &ea, const float2 *U) {
  PipeArgs a{};
  a.W = ea.W;
  a.bias = ea.bias;
  a.out = ea.out;
  a.pre_out = ea.pre_out;
  a.err = L.err;
  a.Ci = ea.Ci;
  a.Co = ea.Co;
  a.act = ea.act;
  a.img = ea.img;
  const bool has_x = mode == EPI_BLOCK_FWD;
  launch_begin(L);
  cudaError_t err;
  if (dtype == DT_F32)
    err = has_x ? launch_pipe_img<float, true>(L, g, a, ea.x, U)
                : launch_pipe_img<float, false>(L, g, a, ea.x, U);
  else if (dtype == DT_F16)
    err = has_x ? launch_pipe_img<__half, true>(L, g, a, ea.x, U)
                : launch_pipe_img<__half, false>(L, g, a, ea.x, U);
  else
    err = has_x ? launch_pipe_img<__nv_bfloat16, true>(L, g, a, ea.x, U)
                : launch_pipe_img<__nv_bfloat16, false>(L, g, a, ea.x, U);
  launch_end(L, has_x ? "epi_block_fwd_pipe" : "epi_spec_pipe");
  return err;
}


bool epi_bwd_pipe_supported(const Geom &g, int dtype, int Ci, int Co, int tanh_pre,
                            const void *x, const void *dy, const void *pre, int act,
                            const void *U) {
  if (dtype == DT_F32 || tanh_pre || g.d < 2) return false;
  if (Ci % 16 != 0 || Co % 16 != 0 || Ci > 64 || Co > 64) return false;
  if (!(g.NL % ROWS == 0 || ROWS % g.NL == 0)) return false;
  const long long SN = (long long)g.S * g.NL;
  if (SN % ROWS != 0 || SN > (1LL << 30) || g.B > (1LL << 30)) return false;
  const BwdGeom e = bwd_geom(g, Ci, Co, act != 0);
  if (e.KS % 4 != 0 || e.KS > 256 || e.used_cols > 512) return false;
  if (e.NS < 2 || e.total > kSmemMax) return false;
  const uintptr_t al = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy) |
                       reinterpret_cast<uintptr_t>(U) | (act ? reinterpret_cast<uintptr_t>(pre) : 0);
  return (al & 15) == 0;
}

cudaError_t launch_epi_bwd_pipe(const Launch &L, const Geom &g, int dtype, const EpiArgs &ea,
                                const float2 *U, int *nparts) {
  PipeArgs a{};
  a.W = ea.W;
  a.out = ea.out;
  a.err = L.err;
  a.Ci = ea.Ci;
  a.Co = ea.Co;
  a.act = ea.act;
  launch_begin(L);
  cudaError_t err = dtype == DT_F16
                        ? launch_bwd_pipe_t<__half>(L, g, a, ea.x, ea.dy, ea.pre, U, ea.partial, nparts)
                        : launch_bwd_pipe_t<__nv_bfloat16>(L, g, a, ea.x, ea.dy, ea.pre, U,
                                                           ea.partial, nparts);
  launch_end(L, "epi_block_bwd_pipe");
  return err;
}

}  // namespace fno
