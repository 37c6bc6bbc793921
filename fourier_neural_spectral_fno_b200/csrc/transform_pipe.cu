// Forward truncated transform (steps S1-S2) as a warp-specialised, TMA-fed
// tcgen05 pipeline.
//
// A tile is a band of 128 rows of one plane (rows = slab-axis index r, the
// band starting at r_off = 128 band).  Both contractions run on the tensor
// cores:
//   S1  X1[r, j] = sum_n x[r, n] F[j, n]       F[2k] = cos(2 pi k n / N_L),
//                                              F[2k+1] = -sin(2 pi k n / N_L)
//       16-bit storage: A = x straight from the TMA ring (K-major, 128-byte
//       swizzle).  Float32: the staging warps read each chunk row once and put
//       its tf32 head and remainder in tensor memory (A from TMEM keeps the
//       shared-memory port for TMA and F), so the two MMAs per K step are
//       A_head [F_hi; F_lo] and A_rest [F_hi; F_lo] (three significant
//       products, ~21 bits).
//   S2  Z[q, k] = sum_r X1[r, k] exp(-i theta(q, r_off + r)),
//       theta(q, r) = 2 pi kS(q) r / S, as one MMA chain with A = the resident
//       twiddle block [cos_hi; sin_hi; cos_lo; sin_lo](q, r) (r_off = 0) in tensor
//       memory and B = X1 (head and remainder rows) in shared memory; the band
//       phase exp(-i theta(q, r_off)) is applied when Z is read out.
//
//   warp 8       TMA producer: 128-byte column chunks of the tile's 128 rows
//   warps 0-3    staging (thread = row): tanh if asked, tf32 head / remainder
//                into TMEM (float32; the stage is then released at once)
//   warp 9       MMA issuer (S1 of tile j, then S2 of tile j - 1); it waits only
//                on chunk-ready and B2-ready barriers (each mbarrier operation in
//                the issuing thread costs tensor-pipe time), the staging and
//                readout warps fold the buffer-free conditions into those
//   warps 4-7    X1 readout -> B operand of S2; Z readout, band phase, store
//
// Every wait is a bounded mbarrier wait; every role leaves its loop on a
// warp-uniform condition.
#include <string.h>

#include "fno_common.cuh"
#include "fno_kernels.cuh"
#include "tc_util.cuh"
#include "tma_util.cuh"

namespace fno {

namespace {

constexpr int ROWS = 128;
constexpr int NSTAGE_WARPS = 4;          // staging warps 0-3
constexpr int WARP_X1 = 4;               // warps 4-7
constexpr int WARP_TMA = 8;
constexpr int WARP_MMA = 9;
constexpr int THREADS = 10 * 32;
constexpr int MAX_STAGES = 8;
constexpr size_t kSmemMax = 227 * 1024;
constexpr int CHUNK_BYTES = 128;         // one swizzle atom row
constexpr int NABUF = 3;                 // A buffers in TMEM (float32 staging ring)

template <typename T> struct FKind {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int fmt = tc::FMT_F16;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
};
template <> struct FKind<float> {
  static constexpr bool tf32 = true;
  static constexpr int EB = 4;
  static constexpr int fmt = tc::FMT_TF32;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
};
template <> struct FKind<__nv_bfloat16> {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int fmt = tc::FMT_BF16;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};

__host__ __device__ inline int rup(int v, int m) { return (v + m - 1) / m * m; }
__host__ __device__ inline size_t alg(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Plan.  TMEM: D1 x2 [0, 2 DC1), a ring of NA = 3 A buffers (tf32: head +
// remainder, 64 columns each; staging runs up to two chunks ahead of the
// MMAs), A2 (128 columns), one D2 (its readout always precedes the next tile's
// S2, which waits for the B2 that follows that readout).
// Shared memory: the TMA ring (the twiddle tables alias it during set-up), F,
// the padded X1 transpose, B2, the readout exchange, the band phases, barriers.
struct PipeGeom {
  int NP;         // 2 mL padded to 16: rows of F_hi (and of F_lo)
  int DC1;        // D1 columns (tf32: [A F_hi | A F_lo])
  int nch;        // column chunks per row
  int CW;         // elements per chunk
  int NS;         // ring stages
  int x1ld;       // padded row stride (floats) of the X1 transpose
  int col_alo, col_a2, col_d2, cols;
  uint32_t fsbo, b2sbo;
  size_t stage, f, fbytes, t, b2, b2half, red, ph, bar, tbase, total;
};

__host__ __device__ inline PipeGeom fpipe_geom(int S, int NL, int mL, int eb, bool tf32) {
  PipeGeom e;
  e.NP = rup(2 * mL, 16);
  e.DC1 = tf32 ? 2 * e.NP : e.NP;
  e.CW = CHUNK_BYTES / eb;
  e.nch = NL / e.CW;
  e.x1ld = 2 * mL + 1;
  e.col_alo = 2 * e.DC1;
  e.col_a2 = e.col_alo + (tf32 ? NABUF * 64 : 0);
  e.col_d2 = e.col_a2 + ROWS;
  e.cols = 512;
  e.fsbo = (uint32_t)(NL * eb / 16) * 128u;
  e.b2sbo = (uint32_t)(ROWS * 4 / 16) * 128u;     // K = 128 rows of float32
  e.stage = (size_t)ROWS * CHUNK_BYTES;            // 16 KB, 1024-aligned
  e.fbytes = (size_t)(tf32 ? 2 : 1) * e.NP * NL * eb;
  e.b2half = (size_t)e.NP * ROWS * 4;
  const size_t tw = sizeof(float2) * ((size_t)NL + S);
  const size_t fixed = alg(e.fbytes, 1024) + alg(sizeof(float) * ROWS * e.x1ld, 128) +
                       alg(2 * e.b2half, 1024) + sizeof(float) * 2 * 32 * 33 +
                       sizeof(float2) * 32 * 32 + sizeof(uint64_t) * (3 * MAX_STAGES + 16) + 16;
  const size_t room = kSmemMax > fixed ? kSmemMax - fixed : 0;
  size_t ns = room / e.stage;
  if (ns > MAX_STAGES) ns = MAX_STAGES;
  while (ns > 0 && ns * e.stage < tw) --ns;        // ring must hold the set-up tables
  if (ns * e.stage < tw) ns = 0;
  e.NS = (int)ns;
  size_t off = (size_t)e.NS * e.stage;
  e.f = off; off = alg(off + e.fbytes, 1024);
  e.b2 = off; off = alg(off + 2 * e.b2half, 1024);
  e.t = off; off = alg(off + sizeof(float) * ROWS * e.x1ld, 128);
  e.red = off; off += sizeof(float) * 2 * 32 * 33;
  e.ph = off; off += sizeof(float2) * 32 * 32;
  e.bar = off; off += sizeof(uint64_t) * (3 * MAX_STAGES + 16);
  e.tbase = off; off += 16;
  e.total = off < 116 * 1024 ? 116 * 1024 : off;
  return e;
}

// K-major, 128-byte swizzle descriptor (8-row groups 1024 bytes apart)
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc,
                                       uint32_t acc, bool tf32) {
  if (tf32)
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
        : "memory");
}

// named barrier over the four readout warps, and the same barrier as an AND
// vote (keeps their exits uniform: a warp that leaves early would strand the
// others at the next barrier)
__device__ __forceinline__ void x1_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool x1_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

struct FPipeArgs {
  float2 *zpart;     // [nbands][planes][QS][mL]
  int *err;
  long long planes;
  int S, NL, mL, mS, QS, nbands;
};


template <typename T, int LOAD>
__global__ void __launch_bounds__(THREADS, 1)
    k_fwd_pipe(const __grid_constant__ CUtensorMap tmx, FPipeArgs a) {
  using K = FKind<T>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int S = a.S, NL = a.NL, mL = a.mL, QS = a.QS;
  const PipeGeom e = fpipe_geom(S, NL, mL, K::EB, K::tf32);
  unsigned char *fsm = smem + e.f;
  unsigned char *b2 = smem + e.b2;
  float *tx = reinterpret_cast<float *>(smem + e.t);
  float *red = reinterpret_cast<float *>(smem + e.red);
  float2 *ph = reinterpret_cast<float2 *>(smem + e.ph);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + e.bar);
  uint64_t *empty = full + MAX_STAGES;
  uint64_t *cready = empty + MAX_STAGES;
  uint64_t *lofree = cready + MAX_STAGES;   // [NABUF] A buffer free
  uint64_t *d1full = lofree + NABUF;        // [2]
  uint64_t *d1free = d1full + 2;            // [2]
  uint64_t *b2ready = d1free + 2;           // [1]
  uint64_t *s2done = b2ready + 1;           // [2]
  uint64_t *fin = s2done + 2;               // [1] all MMAs of the CTA done
  uint32_t *tbase_s = reinterpret_cast<uint32_t *>(smem + e.tbase);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, e.cols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], K::tf32 ? NSTAGE_WARPS : 1);   // tf32: staging frees it
      tc::mbar_init(&cready[s], NSTAGE_WARPS);
    }
    for (int i = 0; i < NABUF; ++i) tc::mbar_init(&lofree[i], 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&d1full[i], 1);
      tc::mbar_init(&d1free[i], 4);
      tc::mbar_init(&s2done[i], 1);
    }
    tc::mbar_init(b2ready, 4);
    tc::mbar_init(fin, 1);
    tma::fence_barrier_init();
  }
  if (warp == WARP_TMA && lane == 0) tma::prefetch_map(&tmx);
  // set-up tables in the (not yet used) ring: last-axis and slab-axis twiddles
  float2 *twL = reinterpret_cast<float2 *>(smem);
  float2 *twS = twL + NL;
  build_twiddles(twL, NL);
  build_twiddles(twS, S);
  __syncthreads();
  // F (B of S1): rows j < 2 mL hold (cos, -sin)(2 pi (j/2) n / NL), tf32 hi rows
  // [0, NP) and lo rows [NP, 2 NP); K-major core matrices
  for (int i = tid; i < e.NP * NL; i += THREADS) {
    const int j = i / NL, n = i - j * NL;
    float v = 0.f;
    if (j < 2 * mL) {
      const float2 w = twL[mulmod(j >> 1, n, NL)];
      v = (j & 1) ? -w.y : w.x;
    }
    const int kb = n * K::EB;
    const uint32_t off = (uint32_t)(j >> 3) * e.fsbo + (kb >> 4) * 128 + (j & 7) * 16 + (kb & 15);
    if (K::tf32) {
      uint32_t hi, lo;
      tc::split_tf32(v, hi, lo);
      *reinterpret_cast<uint32_t *>(fsm + off) = hi;
      *reinterpret_cast<uint32_t *>(fsm + (size_t)e.NP * NL * 4 + off) = lo;
    } else {
      *reinterpret_cast<T *>(fsm + off) = from_f<T>(v);
    }
  }
  // band phases exp(-i theta(q, 128 band)) -> ph[band][q] = (cos, sin)
  for (int i = tid; i < a.nbands * 32; i += THREADS) {
    const int band = i >> 5, q = i & 31;
    const int ks = QS == 1 ? 0 : kept_k(q < QS ? q : 0, a.mS, S);
    ph[i] = twS[mulmod(ks, (band * ROWS) % S, S)];
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;
  if (warp >= WARP_X1 && warp < WARP_X1 + 4) {
    // A2 in TMEM: lane m = 32 blk + q, column r: blk 0 cos_hi, 1 sin_hi, 2 cos_lo, 3 sin_lo
    const int blk = warp - WARP_X1, q = lane;
    const uint32_t row = tbase + ((uint32_t)(blk * 32) << 16) + e.col_a2;
    const int ks = QS == 1 ? 0 : kept_k(q < QS ? q : 0, a.mS, S);
    int idx = 0;
    for (int c0 = 0; c0 < ROWS; c0 += 16) {
      uint32_t v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 w = twS[idx];
        idx += ks;
        if (idx >= S) idx -= S;
        const float val = (blk & 1) ? w.y : w.x;
        uint32_t hi, lo;
        tc::split_tf32(val, hi, lo);
        v[i] = q < QS ? ((blk & 2) ? lo : hi) : 0u;
      }
      tc::tmem_st16(row + c0, v);
    }
    tc::tmem_wait_st();
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();   // tables consumed: the ring may now be filled
  tc::fence_after_sync();

  const long long ntiles = a.planes * a.nbands;
  const long long per_cta = (ntiles + gridDim.x - 1) / gridDim.x;
  const long long t_begin = blockIdx.x * per_cta;
  const long long t_end = t_begin + per_cta < ntiles ? t_begin + per_cta : ntiles;
  const int ntl = t_begin < t_end ? (int)(t_end - t_begin) : 0;
  const int nch = e.nch;

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ TMA producer
    int g = 0;
    bool ok = true;
    for (int j = 0; j < ntl && ok; ++j) {
      const int row0 = (int)((t_begin + j) * ROWS);
      for (int c = 0; c < nch; ++c, ++g) {
        const int s = g % e.NS;
        const bool w = g < e.NS || tc::mbar_wait(&empty[s], ((g / e.NS) - 1) & 1, a.err);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          tma::arrive_expect_tx(&full[s], (uint32_t)e.stage);
          tma::load_4d(smem + (size_t)s * e.stage, &tmx, &full[s], c * e.CW, row0, 0, 0);
        }
        __syncwarp();
      }
    }
    for (int gg = g - 1; gg >= 0 && gg >= g - e.NS; --gg)   // issued loads land before exit
      tc::mbar_wait(&full[gg % e.NS], (gg / e.NS) & 1, nullptr);
  } else if (warp < NSTAGE_WARPS) {
    // ------------------------------------------------------------ staging
    const int r = tid;                                    // row of the tile / TMEM lane
    const uint32_t lrow = tbase + ((uint32_t)(warp * 32) << 16);
    int g = 0;
    bool ok = true;
    for (int j = 0; j < ntl && ok; ++j) {
      for (int c = 0; c < nch; ++c, ++g) {
        const int s = g % e.NS;
        bool w = tc::mbar_wait(&full[s], (g / e.NS) & 1, a.err);
        if (K::tf32 && w && g >= NABUF)
          w = tc::mbar_wait(&lofree[g % NABUF], ((g / NABUF) - 1) & 1, a.err);
        // chunk 0 of tile j also carries "D1 buffer j % 2 is free" to the MMA
        if (w && c == 0 && j >= 2) w = tc::mbar_wait(&d1free[j & 1], ((j - 2) >> 1) & 1, a.err);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (K::tf32 || LOAD == LOAD_TANH) {
          // this row's 128-byte chunk: 16-byte piece p sits at p ^ (r % 8)
          unsigned char *rowp = smem + (size_t)s * e.stage + (size_t)r * CHUNK_BYTES;
          uint4 pc[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) pc[p] = *reinterpret_cast<const uint4 *>(rowp + ((p ^ (r & 7)) << 4));
          if (K::tf32) {
            // head / remainder of the 32 values into A buffer g & 1: head
            // columns [0, 32), remainder [32, 64)
            const uint32_t acol = lrow + e.col_alo + (g % NABUF) * 64;
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
              uint32_t hi[16], lo[16];
#pragma unroll
              for (int p = 0; p < 4; ++p) {
                const uint32_t *u = reinterpret_cast<const uint32_t *>(&pc[hlf * 4 + p]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  float v = __uint_as_float(u[i]);
                  if (LOAD == LOAD_TANH) v = tanhf(v);
                  tc::split_tf32(v, hi[p * 4 + i], lo[p * 4 + i]);
                }
              }
              tc::tmem_st16(acol + hlf * 16, hi);
              tc::tmem_st16(acol + 32 + hlf * 16, lo);
            }
          } else {
#pragma unroll
            for (int p = 0; p < 8; ++p) {
              T *h = reinterpret_cast<T *>(&pc[p]);
#pragma unroll
              for (int i = 0; i < 8; ++i) h[i] = from_f<T>(tanhf(to_f<T>(h[i])));
              *reinterpret_cast<uint4 *>(rowp + ((p ^ (r & 7)) << 4)) = pc[p];
            }
          }
          tc::tmem_wait_st();
          tc::fence_proxy_async_smem();
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          if (K::tf32) tma::arrive(&empty[s]);   // the row data now lives in TMEM
          tma::arrive(&cready[s]);
        }
      }
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t id1 = tc::instr_desc(K::fmt, ROWS, e.DC1);
    const uint32_t id2 = tc::instr_desc(tc::FMT_TF32, ROWS, 2 * e.NP);
    const uint64_t fdesc = tc::smem_desc_kmajor(tc::smem_u32(fsm), 128, e.fsbo);
    const uint64_t b2desc = tc::smem_desc_kmajor(tc::smem_u32(b2), 128, e.b2sbo);
    auto issue_s2 = [&](int jj) -> bool {   // S2 of local tile jj
      // b2ready(jj) follows the readout of D2 for tile jj - 1 in the readout
      // warps' own order, so D2 is free as well
      const bool w = tc::mbar_wait(b2ready, jj & 1, a.err);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc::fence_after_sync();
      if (tc::elect_one()) {   // unrolled: bases plus compile-time offsets
        const uint32_t d2 = tbase + e.col_d2;
        const uint32_t acol = tbase + e.col_a2;
#pragma unroll
        for (int ks = 0; ks < ROWS / 8; ++ks)
          tc::mma_tf32_ts(d2, acol + 8 * ks, b2desc + (uint64_t)(16 * ks), id2, ks > 0 ? 1u : 0u);
        tc::mma_commit(&s2done[jj & 1]);
      }
      __syncwarp();
      return true;
    };
    int g = 0;
    bool ok = true;
    for (int j = 0; j < ntl && ok; ++j) {
      const uint32_t d1 = tbase + (uint32_t)((j & 1) * e.DC1);
      for (int c = 0; c < nch; ++c, ++g) {
        const int s = g % e.NS;
        if (!__all_sync(0xffffffffu, tc::mbar_wait(&cready[s], (g / e.NS) & 1, a.err))) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        if (tc::elect_one()) {
          const uint64_t ad = desc_sw128(tc::smem_u32(smem + (size_t)s * e.stage));
          const uint64_t bd = fdesc + (uint64_t)(c * 4 * 16);
          const uint32_t ahi = tbase + e.col_alo + (g % NABUF) * 64;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint32_t acc = (c | ks) ? 1u : 0u;
            // A: 32 bytes along K inside the swizzle atom; F: 256 bytes per K step
            if (K::tf32) {
              tc::mma_tf32_ts(d1, ahi + ks * 8, bd + (uint64_t)(16 * ks), id1, acc);
              tc::mma_tf32_ts(d1, ahi + 32 + ks * 8, bd + (uint64_t)(16 * ks), id1, 1u);
            } else {
              mma_ss(d1, ad + (uint64_t)(2 * ks), bd + (uint64_t)(16 * ks), id1, acc, false);
            }
          }
          if (K::tf32) tc::mma_commit(&lofree[g % NABUF]);   // A buffer free
          else tc::mma_commit(&empty[s]);                 // stage free
          if (c == nch - 1) tc::mma_commit(&d1full[j & 1]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (j >= 1 && !issue_s2(j - 1)) ok = false;
    }
    if (ok && ntl > 0) ok = issue_s2(ntl - 1);
    // no MMA may still run when TMEM is freed: one last commit covers them all
    if (lane == 0) tc::mma_commit(fin);
    __syncwarp();
    tc::mbar_wait(fin, 0, nullptr);
  } else {
    // ------------------------------------------------------------ X1 / Z warps
    const int blk = warp - WARP_X1;                 // lane quarter
    const int r = blk * 32 + lane;                  // tile row (S1 readout) / A2 row (S2)
    const uint32_t lrow = tbase + ((uint32_t)(blk * 32) << 16);
    const int two_ml = 2 * mL;
    auto readout_s2 = [&](int jj) -> bool {         // Z of local tile jj
      if (!x1_all(tc::mbar_wait(&s2done[jj & 1], (jj >> 1) & 1, a.err))) return false;
      tc::fence_after_sync();
      const uint32_t d2 = lrow + e.col_d2;
      float val[32];
#pragma unroll
      for (int c0 = 0; c0 < 32; c0 += 16) {
        if (c0 >= two_ml) break;
        uint32_t hv[16], lv[16];
        tc::tmem_ld16(d2 + c0, hv);
        tc::tmem_ld16(d2 + e.NP + c0, lv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c0 + i < 32) val[c0 + i] = __uint_as_float(hv[i]) + __uint_as_float(lv[i]);
      }
      tc::fence_before_sync();
      __syncwarp();
      // cos rows = blk 0 (+ blk 2), sin rows = blk 1 (+ blk 3)
      if (blk >= 2) {
#pragma unroll
        for (int n = 0; n < 32; ++n)
          if (n < two_ml) red[((blk - 2) * 32 + lane) * 33 + n] = val[n];
      }
      x1_sync();
      if (blk < 2) {
#pragma unroll
        for (int n = 0; n < 32; ++n)
          if (n < two_ml) val[n] += red[(blk * 32 + lane) * 33 + n];
      }
      x1_sync();
      if (blk == 1) {
#pragma unroll
        for (int n = 0; n < 32; ++n)
          if (n < two_ml) red[lane * 33 + n] = val[n];
      }
      x1_sync();
      if (blk == 0 && lane < QS) {
        const long long tile = t_begin + jj;
        const long long plane = tile / a.nbands;
        const int band = (int)(tile - plane * a.nbands);
        const float2 w = ph[band * 32 + lane];      // exp(-i phi) = (w.x, -w.y)
        float2 *dst = a.zpart + (((long long)band * a.planes + plane) * QS + lane) * mL;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          if (k < mL) {
            const float sr = red[lane * 33 + 2 * k], si = red[lane * 33 + 2 * k + 1];
            const float zr = val[2 * k] + si, zi = val[2 * k + 1] - sr;
            dst[k] = make_float2(w.x * zr + w.y * zi, w.x * zi - w.y * zr);
          }
        }
      }
      x1_sync();   // red is rewritten by the next readout
      return true;
    };
    bool ok = true;
    for (int j = 0; j < ntl && ok; ++j) {
      if (!x1_all(tc::mbar_wait(&d1full[j & 1], (j >> 1) & 1, a.err))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const uint32_t d1 = lrow + (uint32_t)((j & 1) * e.DC1);
      float x1[32];
#pragma unroll
      for (int c0 = 0; c0 < 32; c0 += 16) {
        if (c0 >= two_ml) break;
        uint32_t hv[16];
        tc::tmem_ld16(d1 + c0, hv);
        if (K::tf32) {
          uint32_t lv[16];
          tc::tmem_ld16(d1 + e.NP + c0, lv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < 32) x1[c0 + i] = __uint_as_float(hv[i]) + __uint_as_float(lv[i]);
        } else {
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < 32) x1[c0 + i] = __uint_as_float(hv[i]);
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(&d1free[j & 1]);
#pragma unroll
      for (int n = 0; n < 32; ++n)
        if (n < two_ml) tx[r * e.x1ld + n] = x1[n];
      // B2 is free once S2 of the previous tile has completed
      if (j >= 1) {
        if (!readout_s2(j - 1)) {
          ok = false;
          break;
        }
      } else {
        x1_sync();
      }
      // B2 rows n (tf32 head) and NP + n (remainder), K = tile row; 16-byte
      // chunks of 4 rows, lanes of a quarter warp on 8 distinct rows n
      for (int it = tid - WARP_X1 * 32; it < e.NP * (ROWS / 4); it += 128) {
        const int n = (it & 7) + 8 * ((it >> 3) % (e.NP / 8));
        const int rq = (it >> 3) / (e.NP / 8);
        float v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = n < two_ml ? tx[(rq * 4 + i) * e.x1ld + n] : 0.f;
        uint32_t h[4], l[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) tc::split_tf32(v[i], h[i], l[i]);
        const uint32_t off = (uint32_t)(n >> 3) * e.b2sbo + rq * 128 + (n & 7) * 16;
        *reinterpret_cast<uint4 *>(b2 + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4 *>(b2 + e.b2half + off) = make_uint4(l[0], l[1], l[2], l[3]);
      }
      tc::fence_proxy_async_smem();
      x1_sync();   // tx may be rewritten; every B2 write is done
      if (lane == 0) tma::arrive(b2ready);
    }
    if (ok && ntl > 0) readout_s2(ntl - 1);
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, e.cols);
  }
}

template <typename T, int LOAD>
cudaError_t launch_t(const Launch &L, const Geom &g, long long C, const void *in0,
                     float2 *zpart) {
  using K = FKind<T>;
  const PipeGeom e = fpipe_geom(g.S, g.NL, g.mL, K::EB, K::tf32);
  FPipeArgs a{};
  a.zpart = zpart;
  a.err = L.err;
  a.planes = g.B * C * g.O;
  a.S = g.S;
  a.NL = g.NL;
  a.mL = g.mL;
  a.mS = g.mS;
  a.QS = g.QS;
  a.nbands = g.S / ROWS;
  const long long rows = a.planes * g.S;
  CUtensorMap tmx;
  memset(&tmx, 0, sizeof(tmx));
  const uint64_t dims[4] = {(uint64_t)g.NL, (uint64_t)rows, 1u, 1u};
  const uint64_t rowb = (uint64_t)g.NL * K::EB;
  const uint64_t str[3] = {rowb, rowb * (uint64_t)rows, rowb * (uint64_t)rows};
  const uint32_t box[4] = {(uint32_t)e.CW, (uint32_t)ROWS, 1u, 1u};
  if (!encode_tmap_4d(&tmx, K::tmap, in0, dims, str, box, true)) return cudaErrorInvalidValue;
  const long long ntiles = a.planes * a.nbands;
  const int grid = (int)(ntiles < L.num_sms ? ntiles : L.num_sms);
  auto kern = k_fwd_pipe<T, LOAD>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)e.total);
  kern<<<grid, THREADS, e.total, L.stream>>>(tmx, a);
  return cudaGetLastError();
}

}  // namespace

// Shapes the pipelined transform takes: 128-row bands (S a multiple of 128),
// whole 128-byte column chunks, at most 16 last-axis and 32 slab-axis modes
// (one A2 block of cos/sin x head/remainder rows), TMEM and shared memory fit.
bool fwd_pipe_supported(const Geom &g, int dtype, int load_mode, const void *in0) {
  if (load_mode != LOAD_PLAIN && load_mode != LOAD_TANH) return false;
  const int eb = dtype == DT_F32 ? 4 : 2;
  if (g.S % ROWS != 0 || (g.NL * eb) % CHUNK_BYTES != 0) return false;
  if (g.mL > 16 || g.QS > 32) return false;
  if ((reinterpret_cast<uintptr_t>(in0) & 15) != 0) return false;
  const bool tf32 = dtype == DT_F32;
  const PipeGeom e = fpipe_geom(g.S, g.NL, g.mL, eb, tf32);
  if (e.NS < 2 || e.total > kSmemMax) return false;
  if (e.col_d2 + 2 * e.NP > 512) return false;
  return true;
}

cudaError_t launch_fwd_pipe(const Launch &L, const Geom &g, int dtype, int load_mode,
                            long long C, const void *in0, float2 *zpart) {
  launch_begin(L);
  cudaError_t err;
  const bool th = load_mode == LOAD_TANH;
  if (dtype == DT_F32)
    err = th ? launch_t<float, LOAD_TANH>(L, g, C, in0, zpart)
             : launch_t<float, LOAD_PLAIN>(L, g, C, in0, zpart);
  else if (dtype == DT_F16)
    err = th ? launch_t<__half, LOAD_TANH>(L, g, C, in0, zpart)
             : launch_t<__half, LOAD_PLAIN>(L, g, C, in0, zpart);
  else
    err = th ? launch_t<__nv_bfloat16, LOAD_TANH>(L, g, C, in0, zpart)
             : launch_t<__nv_bfloat16, LOAD_PLAIN>(L, g, C, in0, zpart);
  launch_end(L, "fwd_transform_pipe");
  return err;
}

}  // namespace fno
