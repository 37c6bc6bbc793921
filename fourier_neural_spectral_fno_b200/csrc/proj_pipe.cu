// Projection u = Q2 GELU(Q1 v + q1) + q2 (step S5) as a warp-specialised,
// TMA-fed tcgen05 pipeline.
//
// A tile is 128 consecutive grid points of one sample.  The hidden layer
// h[p, :] = v[p, :] Q1^T is an MMA chain with A = v (point p <-> TMEM lane p)
// and B = Q1 (K-major, resident in shared memory); it never leaves the SM:
// epilogue warps read it from tensor memory, add q1, apply GELU and contract
// with Q2 on the CUDA cores.  Float32 storage: three tf32 passes (v_hi Q1_hi +
// v_hi Q1_lo + v_lo Q1_hi); 16-bit storage: one kind::f16 pass.
//
//   warp 21      TMA producer: v tile [width][128] into ring stage j % NS
//   warps 0-3    staging: v -> A operand in TMEM (tf32 head / remainder)
//   warp 20      MMA issuer: tile j into D buffer j % 2; its one mbarrier wait
//                per tile (aready) also means the D buffer is free, since the
//                staging warps wait for the epilogue before arriving
//   warps 4-19   epilogue: four warps per TMEM lane quarter, each taking a
//                quarter of the hidden units; the quarters' Q2 partial sums
//                meet in shared memory and the first quarter stores u
// Every wait is a bounded mbarrier wait; exits are warp-uniform, and the
// epilogue warps share one named barrier per tile.
#include <string.h>

#include "fno_common.cuh"
#include "fno_kernels.cuh"
#include "tc_util.cuh"
#include "tma_util.cuh"

namespace fno {

namespace {

constexpr int ROWS = 128;
constexpr int NCONV = 4;
constexpr int NEPI = 16;                   // four per TMEM lane quarter
constexpr int NPART = NEPI / 4;            // hidden-unit parts
constexpr int WARP_MMA = NCONV + NEPI;     // 20
constexpr int WARP_TMA = WARP_MMA + 1;     // 21
constexpr int THREADS = (WARP_TMA + 1) * 32;
constexpr int MAX_STAGES = 6;
constexpr int kMaxOut = 4;
constexpr size_t kSmemMax = 227 * 1024;

template <typename T> struct QKind {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int KSTEP = 16;
  static constexpr int fmt = tc::FMT_F16;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
};
template <> struct QKind<float> {
  static constexpr bool tf32 = true;
  static constexpr int EB = 4;
  static constexpr int KSTEP = 8;
  static constexpr int fmt = tc::FMT_TF32;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
};
template <> struct QKind<__nv_bfloat16> {
  static constexpr bool tf32 = false;
  static constexpr int EB = 2;
  static constexpr int KSTEP = 16;
  static constexpr int fmt = tc::FMT_BF16;
  static constexpr CUtensorMapDataType tmap = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};

__host__ __device__ inline int rup(int v, int m) { return (v + m - 1) / m * m; }
__host__ __device__ inline size_t alg(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Plan.  TMEM: two D buffers [0, 2 HP), then two A buffers (tf32: head and
// remainder, 2 Cp columns each).  HP is a multiple of 16 NPART, so every part
// of the hidden units is whole 16-column groups.  Shared memory: the ring (v
// tiles), B = Q1 (head block, then remainder block), q1, Q2, the part-sum
// exchange, barriers.
struct ProjGeom {
  int Cp, HP, ax_cols, col_a, used, NS;
  uint32_t sbo, x_bytes;
  size_t stage, bhalf, b, q1, q2, red, bar, tbase, total;
};

__host__ __device__ inline ProjGeom proj_geom(int width, int hidden, int eb, bool tf32) {
  ProjGeom e;
  e.Cp = rup(width, 16);
  e.HP = rup(hidden, 16 * NPART);
  e.ax_cols = tf32 ? 2 * e.Cp : e.Cp / 2;
  e.col_a = 2 * e.HP;
  e.used = e.col_a + 2 * e.ax_cols;
  e.sbo = (uint32_t)(e.Cp * eb / 16) * 128u;
  e.x_bytes = (uint32_t)(width * ROWS * eb);
  e.stage = alg(e.x_bytes, 1024);
  e.bhalf = (size_t)e.HP * e.Cp * eb;
  const size_t fixed = alg((tf32 ? 2 : 1) * e.bhalf, 1024) + sizeof(float) * e.HP +
                       sizeof(float) * kMaxOut * e.HP +
                       sizeof(float) * 2 * (NPART - 1) * kMaxOut * ROWS +
                       sizeof(uint64_t) * (2 * MAX_STAGES + 8) + 16;
  const size_t room = kSmemMax > fixed ? kSmemMax - fixed : 0;
  const size_t ns = room / e.stage;
  e.NS = (int)(ns < (size_t)MAX_STAGES ? ns : (size_t)MAX_STAGES);
  size_t off = (size_t)e.NS * e.stage;
  e.b = off; off = alg(off + (tf32 ? 2 : 1) * e.bhalf, 1024);
  e.q1 = off; off += sizeof(float) * e.HP;
  e.q2 = off; off += sizeof(float) * kMaxOut * e.HP;
  e.red = off; off += sizeof(float) * 2 * (NPART - 1) * kMaxOut * ROWS;
  off = alg(off, 8);
  e.bar = off; off += sizeof(uint64_t) * (2 * MAX_STAGES + 8);
  e.tbase = off; off += 16;
  e.total = off < 116 * 1024 ? 116 * 1024 : off;
  return e;
}

__host__ __device__ __forceinline__ uint32_t boff(int n, int k, int eb, uint32_t sbo) {
  const int kb = k * eb;
  return (uint32_t)(n >> 3) * sbo + (kb >> 4) * 128 + (n & 7) * 16 + (kb & 15);
}

// named barrier over the epilogue warps
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 512;" ::: "memory"); }
static_assert(NEPI * 32 == 512, "the named barriers count the epilogue threads");
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 512, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

struct ProjArgs {
  const void *Q1, *q1, *Q2, *q2;
  void *u;
  int *err;
  long long B, N;
  int width, hidden, out_ch;
};

// 16 A elements of this thread's lane into TMEM (tf32: head at col, remainder
// at col + lo_off)
template <typename T>
__device__ __forceinline__ void stage16(uint32_t col, uint32_t lo_off, const float (&v)[16]) {
  if (QKind<T>::tf32) {
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) tc::split_tf32(v[i], hi[i], lo[i]);
    tc::tmem_st16(col, hi);
    tc::tmem_st16(col + lo_off, lo);
  } else {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      pk[i] = QKind<T>::fmt == tc::FMT_BF16 ? tc::pack_bf16(v[2 * i], v[2 * i + 1])
                                             : tc::pack_f16(v[2 * i], v[2 * i + 1]);
    tc::tmem_st8(col, pk);
  }
}

// K steps [k0, k0 + NSTEP) of the hidden-layer chain (tf32: v_hi Q1_hi,
// v_hi Q1_lo, v_lo Q1_hi per step); the first step of the chain (k0 = 0)
// overwrites D.
template <typename K, int NSTEP>
__device__ __forceinline__ void proj_steps(uint32_t d, uint32_t a0, int cp, uint64_t bh0,
                                           uint64_t bl0, uint32_t idesc, int k0) {
#pragma unroll
  for (int s = 0; s < NSTEP; ++s) {
    const int ks = k0 + s;
    const uint32_t acc = ks > 0 ? 1u : 0u;
    const uint64_t bo = (uint64_t)(16 * ks);
    if (K::tf32) {
      tc::mma_tf32_ts(d, a0 + 8 * ks, bh0 + bo, idesc, acc);
      tc::mma_tf32_ts(d, a0 + 8 * ks, bl0 + bo, idesc, 1u);
      tc::mma_tf32_ts(d, a0 + (uint32_t)cp + 8 * ks, bh0 + bo, idesc, 1u);
    } else {
      tc::mma_f16_ts(d, a0 + 8 * ks, bh0 + bo, idesc, acc);
    }
  }
}

template <typename T, int CX>
__global__ void __launch_bounds__(THREADS, 1)
    k_proj_pipe(const __grid_constant__ CUtensorMap tmv, ProjArgs a) {
  using K = QKind<T>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int width = a.width, hidden = a.hidden, out_ch = a.out_ch;
  const ProjGeom e = proj_geom(width, hidden, K::EB, K::tf32);
  unsigned char *bsm = smem + e.b;
  float *q1s = reinterpret_cast<float *>(smem + e.q1);
  float *q2s = reinterpret_cast<float *>(smem + e.q2);
  float *red = reinterpret_cast<float *>(smem + e.red);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + e.bar);
  uint64_t *empty = full + MAX_STAGES;
  uint64_t *aready = empty + MAX_STAGES;   // [2]
  uint64_t *mdone = aready + 2;            // [2]
  uint64_t *dempty = mdone + 2;            // [2]
  uint64_t *fin = dempty + 2;              // [1]
  uint32_t *tbase_s = reinterpret_cast<uint32_t *>(smem + e.tbase);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long N = a.N;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, 512);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], NCONV);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aready[i], NCONV);
      tc::mbar_init(&mdone[i], 1);
      tc::mbar_init(&dempty[i], NEPI);
    }
    tc::mbar_init(fin, 1);
    tma::fence_barrier_init();
  }
  if (warp == WARP_TMA && lane == 0) tma::prefetch_map(&tmv);
  for (size_t i = (size_t)tid * 16; i < (K::tf32 ? 2 : 1) * e.bhalf; i += THREADS * 16)
    *reinterpret_cast<uint4 *>(bsm + i) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  {  // B = Q1 [hidden][width] (head rows block, remainder block), q1, Q2
    const T *Q1 = reinterpret_cast<const T *>(a.Q1);
    const int nq = hidden * width;
    for (int i0 = tid; i0 < nq; i0 += 8 * THREADS) {   // eight loads in flight
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = i0 + u * THREADS < nq ? to_f<T>(Q1[i0 + u * THREADS]) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * THREADS;
        if (i >= nq) break;
        const int h = i / width, c = i - h * width;
        const uint32_t o = boff(h, c, K::EB, e.sbo);
        if (K::tf32) {
          uint32_t hi, lo;
          tc::split_tf32(v[u], hi, lo);
          *reinterpret_cast<uint32_t *>(bsm + o) = hi;
          *reinterpret_cast<uint32_t *>(bsm + e.bhalf + o) = lo;
        } else {
          *reinterpret_cast<T *>(bsm + o) = from_f<T>(v[u]);
        }
      }
    }
    const T *q1 = reinterpret_cast<const T *>(a.q1);
    const T *Q2 = reinterpret_cast<const T *>(a.Q2);
    for (int h = tid; h < e.HP; h += THREADS) q1s[h] = h < hidden ? to_f<T>(q1[h]) : 0.f;
    for (int i = tid; i < kMaxOut * e.HP; i += THREADS) {
      const int o = i / e.HP, h = i - o * e.HP;
      q2s[i] = (o < out_ch && h < hidden) ? 0.5f * to_f<T>(Q2[o * hidden + h]) : 0.f;
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;

  const long long tpb = N / ROWS;
  const long long ntiles = a.B * tpb;
  const long long per_cta = (ntiles + gridDim.x - 1) / gridDim.x;
  const long long t_begin = blockIdx.x * per_cta;
  const long long t_end = t_begin + per_cta < ntiles ? t_begin + per_cta : ntiles;
  const int ntl = t_begin < t_end ? (int)(t_end - t_begin) : 0;

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ TMA producer
    int j = 0;
    for (; j < ntl; ++j) {
      const int s = j % e.NS;
      const bool w = j < e.NS || tc::mbar_wait(&empty[s], ((j / e.NS) - 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, w)) break;
      if (lane == 0) {
        const long long tile = t_begin + j;
        const long long b = tile / tpb;
        const int n0 = (int)((tile - b * tpb) * ROWS);
        tma::arrive_expect_tx(&full[s], e.x_bytes);
        tma::load_4d(smem + (size_t)s * e.stage, &tmv, &full[s], n0, 0, 0, (int)b);
      }
      __syncwarp();
    }
    for (int jj = j - 1; jj >= 0 && jj >= j - e.NS; --jj)
      tc::mbar_wait(&full[jj % e.NS], (jj / e.NS) & 1, nullptr);
  } else if (warp < NCONV) {
    // ------------------------------------------------------------ staging
    const int t = tid;
    const uint32_t arow = tbase + ((uint32_t)(warp * 32) << 16);
    const uint32_t lo_off = K::tf32 ? (uint32_t)e.Cp : 0u;
    for (int j = 0; j < ntl; ++j) {
      const int s = j % e.NS;
      bool w = tc::mbar_wait(&full[s], (j / e.NS) & 1, a.err);
      if (w && j >= 2) w = tc::mbar_wait(&mdone[j & 1], ((j - 2) >> 1) & 1, a.err);
      // aready(j) also carries "D buffer j % 2 is free" to the MMA thread
      if (w && j >= 2) w = tc::mbar_wait(&dempty[j & 1], ((j - 2) >> 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, w)) break;
      tc::fence_after_sync();
      const T *xs = reinterpret_cast<const T *>(smem + (size_t)s * e.stage);
      const uint32_t ac = arow + e.col_a + (j & 1) * e.ax_cols;
#pragma unroll
      for (int c0 = 0; c0 < CX; c0 += 16) {
        if (c0 < e.Cp) {
          float vals[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) vals[i] = c0 + i < width ? to_f<T>(xs[(c0 + i) * ROWS + t]) : 0.f;
          stage16<T>(ac + (K::tf32 ? c0 : c0 / 2), lo_off, vals);
        }
      }
      __syncwarp();
      if (lane == 0) tma::arrive(&empty[s]);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(&aready[j & 1]);
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = tc::instr_desc(K::fmt, ROWS, e.HP);
    const uint64_t bh0 = tc::smem_desc_kmajor(tc::smem_u32(bsm), 128, e.sbo);
    const uint64_t bl0 = tc::smem_desc_kmajor(tc::smem_u32(bsm + e.bhalf), 128, e.sbo);
    const int ns = e.Cp / K::KSTEP;
    for (int j = 0; j < ntl; ++j) {
      const bool w = tc::mbar_wait(&aready[j & 1], (j >> 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, w)) break;
      tc::fence_after_sync();
      // one elected thread issues the K steps: the exact unrolled sequence for
      // the common widths, else a plain loop (operands advance by 8 TMEM
      // columns and 256 bytes of B per step)
      if (tc::elect_one()) {
        const uint32_t d = tbase + (uint32_t)((j & 1) * e.HP);
        const uint32_t a0 = tbase + e.col_a + (j & 1) * e.ax_cols;
        switch (ns) {
          case 1: proj_steps<K, 1>(d, a0, e.Cp, bh0, bl0, idesc, 0); break;
          case 2: proj_steps<K, 2>(d, a0, e.Cp, bh0, bl0, idesc, 0); break;
          case 3: proj_steps<K, 3>(d, a0, e.Cp, bh0, bl0, idesc, 0); break;
          case 4: proj_steps<K, 4>(d, a0, e.Cp, bh0, bl0, idesc, 0); break;
          case 6: proj_steps<K, 6>(d, a0, e.Cp, bh0, bl0, idesc, 0); break;
          case 8: proj_steps<K, 8>(d, a0, e.Cp, bh0, bl0, idesc, 0); break;
          default:
            for (int ks = 0; ks < ns; ++ks) proj_steps<K, 1>(d, a0, e.Cp, bh0, bl0, idesc, ks);
        }
        tc::mma_commit(&mdone[j & 1]);
      }
      __syncwarp();
    }
    if (lane == 0) tc::mma_commit(fin);   // covers every MMA this CTA issued
    __syncwarp();
    tc::mbar_wait(fin, 0, nullptr);
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, part = (warp - NCONV) >> 2;
    const int t = q * 32 + lane;
    const uint32_t arow = tbase + ((uint32_t)(q * 32) << 16);
    const int hbeg = part * (e.HP / NPART), hend = hbeg + e.HP / NPART;
    T *u = reinterpret_cast<T *>(a.u);
    const T *q2 = reinterpret_cast<const T *>(a.q2);
    float q2b[kMaxOut];
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o) q2b[o] = o < out_ch ? to_f<T>(q2[o]) : 0.f;
    // 16 hidden units h0.. of this point: + q1, GELU, into the Q2 sums
    auto group = [&](const uint32_t (&dv)[16], int h0, float (&acc)[kMaxOut]) {
#pragma unroll
      for (int i = 0; i < 16; i += 4) {   // q1 / Q2 as 16-byte vectors
        const float4 qa = *reinterpret_cast<const float4 *>(q1s + h0 + i);
        float z0 = __uint_as_float(dv[i]) + qa.x;
        float z1 = __uint_as_float(dv[i + 1]) + qa.y;
        float z2 = __uint_as_float(dv[i + 2]) + qa.z;
        float z3 = __uint_as_float(dv[i + 3]) + qa.w;
        gelu2_dbl(z0, z1);   // 2 GELU: q2s holds Q2 / 2
        gelu2_dbl(z2, z3);
#pragma unroll
        for (int o = 0; o < kMaxOut; ++o) {
          if (o < out_ch) {
            const float4 qb = *reinterpret_cast<const float4 *>(q2s + o * e.HP + h0 + i);
            acc[o] = fmaf(qb.w, z3, fmaf(qb.z, z2, fmaf(qb.y, z1, fmaf(qb.x, z0, acc[o]))));
          }
        }
      }
    };
    for (int j = 0; j < ntl; ++j) {
      if (!epi_all(tc::mbar_wait(&mdone[j & 1], (j >> 1) & 1, a.err))) break;
      tc::fence_after_sync();
      const uint32_t dcol = arow + (uint32_t)((j & 1) * e.HP);
      float acc[kMaxOut];
#pragma unroll
      for (int o = 0; o < kMaxOut; ++o) acc[o] = 0.f;
      // rounds of two 16-column groups: both loads in flight, one wait; the
      // last round's wait frees the D buffer
      for (int r0 = hbeg; r0 < hend; r0 += 32) {
        const bool two = r0 + 16 < hend;            // warp-uniform
        uint32_t dv0[16], dv1[16];
        tc::tmem_ld16(dcol + r0, dv0);
        if (two) tc::tmem_ld16(dcol + r0 + 16, dv1);
        tc::tmem_wait_ld();
        if (r0 + 32 >= hend) {
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tma::arrive(&dempty[j & 1]);
        }
        group(dv0, r0, acc);
        if (two) group(dv1, r0 + 16, acc);
      }
      // parts 1.. leave their sums in buffer j % 2; part 0 adds them and stores
      float *rb = red + (j & 1) * (NPART - 1) * kMaxOut * ROWS;
      if (part > 0) {
#pragma unroll
        for (int o = 0; o < kMaxOut; ++o)
          if (o < out_ch) rb[((part - 1) * kMaxOut + o) * ROWS + t] = acc[o];
      }
      epi_sync();
      if (part == 0) {
        const long long tile = t_begin + j;
        const long long b = tile / tpb;
        const long long n = (tile - b * tpb) * ROWS + t;
#pragma unroll
        for (int o = 0; o < kMaxOut; ++o) {
          if (o < out_ch) {
            float v = acc[o] + q2b[o];
#pragma unroll
            for (int p2 = 0; p2 < NPART - 1; ++p2) v += rb[(p2 * kMaxOut + o) * ROWS + t];
            u[(b * out_ch + o) * N + n] = from_f<T>(v);
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, 512);
  }
}

template <typename T>
cudaError_t launch_t(const Launch &L, const Geom &g, const ProjArgs &a, const void *v) {
  using K = QKind<T>;
  const ProjGeom e = proj_geom(a.width, a.hidden, K::EB, K::tf32);
  CUtensorMap tmv;
  memset(&tmv, 0, sizeof(tmv));
  const uint64_t dims[4] = {(uint64_t)g.N, 1u, (uint64_t)a.width, (uint64_t)g.B};
  const uint64_t rowb = (uint64_t)g.N * K::EB;
  const uint64_t str[3] = {rowb, rowb, rowb * (uint64_t)a.width};
  const uint32_t box[4] = {(uint32_t)ROWS, 1u, (uint32_t)a.width, 1u};
  if (!encode_tmap_4d(&tmv, K::tmap, v, dims, str, box)) return cudaErrorInvalidValue;
  const long long ntiles = g.B * (g.N / ROWS);
  const int grid = (int)(ntiles < L.num_sms ? ntiles : L.num_sms);
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)e.total);
    kern<<<grid, THREADS, e.total, L.stream>>>(tmv, a);
  };
  if (a.width <= 16) go(k_proj_pipe<T, 16>);
  else if (a.width <= 32) go(k_proj_pipe<T, 32>);
  else go(k_proj_pipe<T, 64>);
  return cudaGetLastError();
}

// ===========================================================================
// Projection backward (16-bit storage, hidden <= 128) as a tcgen05 pipeline.
// For a tile of 128 consecutive points p of one sample:
//   z = v Q1^T + q1, g = GELU(z), dh = (du Q2) GELU'(z)
//   dv = dh Q1;  dQ1 += dh^T v, dq1 += sum dh;  dQ2 += du^T g, dq2 += sum du
// Four MMA chains: (1) Z = v Q1^T (A = v staged into TMEM, B = Q1 resident),
// (2) [dQ1 | dq1] += dh^T [v; 1] (A = dh^T in shared memory, B = the v tile
// straight from the ring stage: TMA boxes with 128-byte swizzle followed by
// sixteen rows of ones), (3) dv = dh Q1 (A = dh in TMEM, B = Q1^T resident,
// written over the tile's Z buffer), (4) dQ2^T += g^T du (A = g^T, B = du).
// The epilogue warps evaluate GELU and GELU' between chain (1) and the rest.
//
//   warp 21      TMA: v (two swizzled 64-point boxes) and du of tile j
//   warps 0-3    staging: v -> A_v (TMEM), from the swizzled boxes
//   warp 20      MMA: chain (1) of tile j, then chains (3), (2), (4) of j - 1
//   warps 4-19   epilogue (four per TMEM lane quarter, a quarter of the hidden
//                units each): z -> dh, g -> A_dh, dh^T, g^T, du; then dv of
//                the previous tile from TMEM to global; at the end the dQ1 /
//                dQ2 accumulators -> per-CTA partials
// ===========================================================================
constexpr int PB_STAGES = 4;
constexpr int PB_XBOX = 64;

struct PbGeom {
  int Cw, HP, NWq, NS;
  int col_z, col_av, col_ah, col_q1, col_q2, used, cols;
  uint32_t sbo_q1, sbo_q1t, sbo_t, bytes_tx;
  size_t xbox, du_off, stage, bq1, bq1t, adht, agt, bdu, q1s, q2s, dq2, bar, tbase, total;
};

__host__ __device__ inline PbGeom pb_geom(int width, int out_ch) {
  PbGeom e;
  e.Cw = width;                   // multiple of 16
  e.HP = ROWS;                    // hidden padded to 128 (the M of chains 2 and 4)
  e.NWq = width + 16;             // N of chain (2): v rows, then ones
  e.col_z = 0;                    // two Z / dv buffers
  e.col_av = 2 * e.HP;
  e.col_ah = e.col_av + width;    // two A_v buffers of width / 2 columns
  e.col_q1 = e.col_ah + e.HP / 2;
  e.col_q2 = e.col_q1 + rup(e.NWq, 16);
  e.used = e.col_q2 + 16;
  e.cols = 32;
  while (e.cols < e.used && e.cols < 1024) e.cols *= 2;
  e.sbo_q1 = (uint32_t)(width * 2 / 16) * 128u;     // B of (1): rows h, K = c
  e.sbo_q1t = (uint32_t)(e.HP * 2 / 16) * 128u;     // B of (3): rows c, K = h
  e.sbo_t = (uint32_t)(ROWS * 2 / 16) * 128u;       // K = 128 points
  e.xbox = (size_t)e.NWq * 128;
  e.du_off = 2 * e.xbox;
  e.stage = alg(e.du_off + (size_t)kMaxOut * ROWS * 2, 1024);
  e.bytes_tx = (uint32_t)(2 * (size_t)width * 128 + (size_t)out_ch * ROWS * 2);
  size_t off = 0;
  const size_t fixed = alg((size_t)e.HP * width * 2, 1024) + alg((size_t)width * e.HP * 2, 1024) +
                       2 * (size_t)ROWS * ROWS * 2 + (size_t)16 * ROWS * 2 +
                       sizeof(float) * (e.HP + kMaxOut * e.HP + 8) +
                       sizeof(uint64_t) * (2 * PB_STAGES + 12) + 16 + 1024;
  const size_t room = kSmemMax > fixed ? kSmemMax - fixed : 0;
  const size_t ns = room / e.stage;
  e.NS = (int)(ns < (size_t)PB_STAGES ? ns : (size_t)PB_STAGES);
  off = (size_t)(e.NS > 0 ? e.NS : 0) * e.stage;
  e.bq1 = off; off = alg(off + (size_t)e.HP * width * 2, 1024);
  e.bq1t = off; off = alg(off + (size_t)width * e.HP * 2, 1024);
  e.adht = off; off += (size_t)ROWS * ROWS * 2;
  e.agt = off; off += (size_t)ROWS * ROWS * 2;
  e.bdu = off; off += (size_t)16 * ROWS * 2;
  e.q1s = off; off += sizeof(float) * e.HP;
  e.q2s = off; off += sizeof(float) * kMaxOut * e.HP;
  e.dq2 = off; off += sizeof(float) * 8;
  off = alg(off, 8);
  e.bar = off; off += sizeof(uint64_t) * (2 * PB_STAGES + 12);
  e.tbase = off; off += 16;
  e.total = off < 116 * 1024 ? 116 * 1024 : off;
  return e;
}

__device__ __forceinline__ uint64_t pb_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// byte offset of element (row c, point pp < 64) in a 128-byte-swizzled box
__device__ __forceinline__ uint32_t sw128_off(int c, int pp) {
  const int byte = pp * 2;
  return (uint32_t)(c * 128 + ((((byte >> 4) ^ (c & 7)) & 7) << 4) + (byte & 15));
}

template <typename T, int CX>
__global__ void __launch_bounds__(THREADS, 1)
    k_proj_bwd_pipe(const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdu,
                    ProjArgs a, void *dv_out, float *partial) {
  using K = QKind<T>;
  static_assert(!QKind<T>::tf32, "16-bit storage only");
  extern __shared__ __align__(1024) unsigned char smem[];
  const int width = a.width, hidden = a.hidden, out_ch = a.out_ch;
  const PbGeom e = pb_geom(width, out_ch);
  unsigned char *bq1 = smem + e.bq1;
  unsigned char *bq1t = smem + e.bq1t;
  unsigned char *adht = smem + e.adht;
  unsigned char *agt = smem + e.agt;
  unsigned char *bdu = smem + e.bdu;
  float *q1s = reinterpret_cast<float *>(smem + e.q1s);
  float *q2s = reinterpret_cast<float *>(smem + e.q2s);
  float *dq2s = reinterpret_cast<float *>(smem + e.dq2);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + e.bar);
  uint64_t *empty = full + PB_STAGES;
  uint64_t *aready = empty + PB_STAGES;   // [2]
  uint64_t *zdone = aready + 2;           // [2]
  uint64_t *zfree = zdone + 2;            // [2]
  uint64_t *hready = zfree + 2;           // [1]
  uint64_t *hdone = hready + 1;           // [1]
  uint64_t *fin = hdone + 1;              // [1]
  uint32_t *tbase_s = reinterpret_cast<uint32_t *>(smem + e.tbase);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long N = a.N;

  if (warp == 0) {
    tc::tmem_alloc(tbase_s, e.cols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < PB_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&aready[i], NCONV);
      tc::mbar_init(&zdone[i], 1);
      tc::mbar_init(&zfree[i], NEPI);
    }
    tc::mbar_init(hready, NEPI);
    tc::mbar_init(hdone, 1);
    tc::mbar_init(fin, 1);
    tma::fence_barrier_init();
  }
  if (warp == WARP_TMA && lane == 0) {
    tma::prefetch_map(&tmv);
    tma::prefetch_map(&tmdu);
  }
  // zero the resident operands (padded rows stay zero), ones rows of the boxes
  for (size_t i = (size_t)tid * 16; i < e.q1s - e.bq1; i += THREADS * 16)
    *reinterpret_cast<uint4 *>(bq1 + i) = make_uint4(0, 0, 0, 0);
  {
    const uint32_t one2 = QKind<T>::fmt == tc::FMT_BF16 ? 0x3F803F80u : 0x3C003C00u;
    const int per_box = 16 * 128 / 16;
    for (int i = tid; i < e.NS * 2 * per_box; i += THREADS) {
      const int sb = i / per_box, c = i - sb * per_box;
      unsigned char *dst = smem + (size_t)(sb >> 1) * e.stage + (size_t)(sb & 1) * e.xbox +
                           (size_t)width * 128 + (size_t)c * 16;
      *reinterpret_cast<uint4 *>(dst) = make_uint4(one2, one2, one2, one2);
    }
  }
  __syncthreads();
  {  // Q1 [hidden][width] -> B of (1) (rows h, K = c) and B of (3) (rows c, K = h)
    const T *Q1 = reinterpret_cast<const T *>(a.Q1);
    for (int i = tid; i < hidden * width; i += THREADS) {
      const int h = i / width, c = i - h * width;
      *reinterpret_cast<T *>(bq1 + boff(h, c, 2, e.sbo_q1)) = Q1[i];
      *reinterpret_cast<T *>(bq1t + boff(c, h, 2, e.sbo_q1t)) = Q1[i];
    }
    const T *q1 = reinterpret_cast<const T *>(a.q1);
    const T *Q2 = reinterpret_cast<const T *>(a.Q2);
    for (int h = tid; h < e.HP; h += THREADS) q1s[h] = h < hidden ? to_f<T>(q1[h]) : 0.f;
    for (int i = tid; i < kMaxOut * e.HP; i += THREADS) {
      const int o = i / e.HP, h = i - o * e.HP;
      q2s[i] = (o < out_ch && h < hidden) ? to_f<T>(Q2[o * hidden + h]) : 0.f;
    }
    if (tid < 8) dq2s[tid] = 0.f;
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tbase_s;

  const long long tpb = N / ROWS;
  const long long ntiles = a.B * tpb;
  const long long per_cta = (ntiles + gridDim.x - 1) / gridDim.x;
  const long long t_begin = blockIdx.x * per_cta;
  const long long t_end = t_begin + per_cta < ntiles ? t_begin + per_cta : ntiles;
  const int ntl = t_begin < t_end ? (int)(t_end - t_begin) : 0;

  if (warp == WARP_TMA) {
    // ------------------------------------------------------------ TMA producer
    int j = 0;
    for (; j < ntl; ++j) {
      const int s = j % e.NS;
      const bool w = j < e.NS || tc::mbar_wait(&empty[s], ((j / e.NS) - 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, w)) break;
      if (lane == 0) {
        const long long tile = t_begin + j;
        const long long b = tile / tpb;
        const int n0 = (int)((tile - b * tpb) * ROWS);
        unsigned char *st = smem + (size_t)s * e.stage;
        tma::arrive_expect_tx(&full[s], e.bytes_tx);
        tma::load_4d(st, &tmv, &full[s], n0, 0, 0, (int)b);
        tma::load_4d(st + e.xbox, &tmv, &full[s], n0 + PB_XBOX, 0, 0, (int)b);
        tma::load_4d(st + e.du_off, &tmdu, &full[s], n0, 0, 0, (int)b);
      }
      __syncwarp();
    }
    for (int jj = j - 1; jj >= 0 && jj >= j - e.NS; --jj)
      tc::mbar_wait(&full[jj % e.NS], (jj / e.NS) & 1, nullptr);
  } else if (warp < NCONV) {
    // ------------------------------------------------------------ staging
    const int t = tid;
    const uint32_t arow = tbase + ((uint32_t)(warp * 32) << 16);
    const int box = t / PB_XBOX, pp = t - box * PB_XBOX;
    for (int j = 0; j < ntl; ++j) {
      const int s = j % e.NS;
      bool w = tc::mbar_wait(&full[s], (j / e.NS) & 1, a.err);
      if (w && j >= 2) w = tc::mbar_wait(&zdone[j & 1], ((j - 2) >> 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, w)) break;
      tc::fence_after_sync();
      const unsigned char *xs = smem + (size_t)s * e.stage + (size_t)box * e.xbox;
      const uint32_t ac = arow + e.col_av + (j & 1) * (width / 2);
#pragma unroll
      for (int c0 = 0; c0 < CX; c0 += 16) {
        if (c0 < width) {
          float vals[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            vals[i] = to_f<T>(*reinterpret_cast<const T *>(xs + sw128_off(c0 + i, pp)));
          stage16<T>(ac + c0 / 2, 0u, vals);
        }
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(&aready[j & 1]);
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t id1 = tc::instr_desc(K::fmt, ROWS, e.HP);
    const uint32_t id3 = tc::instr_desc(K::fmt, ROWS, width);
    const uint32_t id2 = tc::instr_desc(K::fmt, ROWS, e.NWq);
    const uint32_t id4 = tc::instr_desc(K::fmt, ROWS, 16);
    const uint64_t b1 = tc::smem_desc_kmajor(tc::smem_u32(bq1), 128, e.sbo_q1);
    const uint64_t b3 = tc::smem_desc_kmajor(tc::smem_u32(bq1t), 128, e.sbo_q1t);
    const uint64_t a2 = tc::smem_desc_kmajor(tc::smem_u32(adht), 128, e.sbo_t);
    const uint64_t a4 = tc::smem_desc_kmajor(tc::smem_u32(agt), 128, e.sbo_t);
    const uint64_t b4 = tc::smem_desc_kmajor(tc::smem_u32(bdu), 128, e.sbo_t);
    const int n1 = width / 16;
    // chains (3), (2), (4) of local tile jj
    auto second = [&](int jj) -> bool {
      const bool w = tc::mbar_wait(hready, jj & 1, a.err);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc::fence_after_sync();
      if (tc::elect_one()) {
        const uint32_t dz = tbase + e.col_z + (jj & 1) * e.HP;
#pragma unroll
        for (int k = 0; k < ROWS / 16; ++k)   // dv = dh Q1 (K = 128 hidden)
          tc::mma_f16_ts(dz, tbase + e.col_ah + 8 * k, b3 + (uint64_t)(16 * k), id3,
                         k > 0 ? 1u : 0u);
        const unsigned char *xs = smem + (size_t)(jj % e.NS) * e.stage;
        const uint64_t x0 = pb_desc_sw128(tc::smem_u32(xs)), x1 = pb_desc_sw128(tc::smem_u32(xs + e.xbox));
#pragma unroll
        for (int k = 0; k < ROWS / 16; ++k)   // [dQ1 | dq1] += dh^T [v; 1]
          tc::mma_f16_ss(tbase + e.col_q1, a2 + (uint64_t)(16 * k),
                         (k < 4 ? x0 : x1) + (uint64_t)(2 * (k & 3)), id2,
                         (jj > 0 || k > 0) ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < ROWS / 16; ++k)   // dQ2^T += g^T du
          tc::mma_f16_ss(tbase + e.col_q2, a4 + (uint64_t)(16 * k), b4 + (uint64_t)(16 * k), id4,
                         (jj > 0 || k > 0) ? 1u : 0u);
        tc::mma_commit(&empty[jj % e.NS]);
        tc::mma_commit(hdone);
      }
      __syncwarp();
      return true;
    };
    int j = 0;
    bool ok = true;
    for (; j < ntl && ok; ++j) {
      bool w = tc::mbar_wait(&aready[j & 1], (j >> 1) & 1, a.err);
      if (w && j >= 2) w = tc::mbar_wait(&zfree[j & 1], ((j - 2) >> 1) & 1, a.err);
      if (!__all_sync(0xffffffffu, w)) break;
      tc::fence_after_sync();
      if (tc::elect_one()) {
        const uint32_t dz = tbase + e.col_z + (j & 1) * e.HP;
        const uint32_t av = tbase + e.col_av + (j & 1) * (width / 2);
        switch (n1) {   // Z = v Q1^T (K = width)
          case 4:
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc::mma_f16_ts(dz, av + 8 * k, b1 + (uint64_t)(16 * k), id1, k > 0 ? 1u : 0u);
            break;
          default:
            for (int k = 0; k < n1; ++k)
              tc::mma_f16_ts(dz, av + 8 * k, b1 + (uint64_t)(16 * k), id1, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&zdone[j & 1]);
      }
      __syncwarp();
      if (j >= 1) ok = second(j - 1);
    }
    if (ok && j == ntl && ntl > 0) ok = second(ntl - 1);
    if (tc::elect_one()) tc::mma_commit(fin);
    __syncwarp();
    tc::mbar_wait(fin, 0, nullptr);
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, part = (warp - NCONV) >> 2;
    const int t = q * 32 + lane;
    const uint32_t arow = tbase + ((uint32_t)(q * 32) << 16);
    const int h0 = part * (e.HP / 4);          // 32 hidden units of this warp
    const int cw = width / 4;                  // dv columns of this warp (multiple of 4)
    T *dv = reinterpret_cast<T *>(dv_out);
    float dq2acc[kMaxOut];
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o) dq2acc[o] = 0.f;
    // dv of local tile jj from its Z buffer to global, then the buffer is free
    auto store_dv = [&](int jj) {
      const long long tile = t_begin + jj;
      const long long b = tile / tpb;
      const long long n = (tile - b * tpb) * ROWS + t;
      const uint32_t dcol = arow + e.col_z + (jj & 1) * e.HP + part * cw;
      for (int c0 = 0; c0 < cw; c0 += 4) {
        uint32_t dd[4];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(dd[0]), "=r"(dd[1]), "=r"(dd[2]), "=r"(dd[3])
                     : "r"(dcol + c0)
                     : "memory");
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dv[(b * width + part * cw + c0 + i) * N + n] = from_f<T>(__uint_as_float(dd[i]));
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(&zfree[jj & 1]);
    };
    int j = 0;
    for (; j < ntl; ++j) {
      if (!epi_all(tc::mbar_wait(&zdone[j & 1], (j >> 1) & 1, a.err))) break;
      tc::fence_after_sync();
      const int s = j % e.NS;
      const T *dus = reinterpret_cast<const T *>(smem + (size_t)s * e.stage + e.du_off);
      float du_t[kMaxOut];
#pragma unroll
      for (int o = 0; o < kMaxOut; ++o) du_t[o] = o < out_ch ? to_f<T>(dus[o * ROWS + t]) : 0.f;
      // z of this warp's 32 hidden units -> g, dh
      float gv[32], dhv[32];
      {
        uint32_t z0[16], z1[16];
        const uint32_t zc = arow + e.col_z + (j & 1) * e.HP + h0;
        tc::tmem_ld16(zc, z0);
        tc::tmem_ld16(zc + 16, z1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int h = h0 + i;
          const float z = __uint_as_float(i < 16 ? z0[i] : z1[i - 16]) + q1s[h];
          float gz, gp;
          gelu_and_grad_f(z, gz, gp);
          float dg = 0.f;
#pragma unroll
          for (int o = 0; o < kMaxOut; ++o)
            if (o < out_ch) dg = fmaf(q2s[o * e.HP + h], du_t[o], dg);
          gv[i] = gz;
          dhv[i] = dg * gp;
        }
      }
      // the previous tile's chains (2)-(4) are done with A_dh, dh^T, g^T, du
      if (j >= 1 && !epi_all(tc::mbar_wait(hdone, (j - 1) & 1, a.err))) break;
      tc::fence_after_sync();
      {
        const uint32_t ah = arow + e.col_ah + h0 / 2;
        float v16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v16[i] = dhv[i];
        stage16<T>(ah, 0u, v16);
#pragma unroll
        for (int i = 0; i < 16; ++i) v16[i] = dhv[16 + i];
        stage16<T>(ah + 8, 0u, v16);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          *reinterpret_cast<T *>(adht + boff(h0 + i, t, 2, e.sbo_t)) = from_f<T>(dhv[i]);
          *reinterpret_cast<T *>(agt + boff(h0 + i, t, 2, e.sbo_t)) = from_f<T>(gv[i]);
        }
        if (part == 0) {
#pragma unroll
          for (int o = 0; o < kMaxOut; ++o) {
            if (o < out_ch) {
              *reinterpret_cast<T *>(bdu + boff(o, t, 2, e.sbo_t)) = from_f<T>(du_t[o]);
              dq2acc[o] += du_t[o];
            }
          }
        }
      }
      tc::tmem_wait_st();
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tma::arrive(hready);
      if (j >= 1) store_dv(j - 1);
    }
    const bool done_all = epi_all(j == ntl);
    if (done_all && ntl > 0) {
      if (epi_all(tc::mbar_wait(hdone, (ntl - 1) & 1, a.err))) {
        tc::fence_after_sync();
        store_dv(ntl - 1);
      }
    }
    // dq2: warp sums of the part-0 warps into shared memory
    if (part == 0) {
#pragma unroll
      for (int o = 0; o < kMaxOut; ++o) {
        float v = dq2acc[o];
        for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
        if (lane == 0 && o < out_ch) atomicAdd(&dq2s[o], v);
      }
    }
    epi_sync();
    tc::fence_after_sync();
    // accumulators -> partials: row h = lane t of the quarter
    float *dst = partial + (long long)blockIdx.x * (hidden * (width + 1) + out_ch * (hidden + 1));
    const bool row = t < hidden && done_all;
    for (int c0 = part * 16; c0 < e.NWq; c0 += 64) {
      uint32_t dd[16];
      tc::tmem_ld16(arow + e.col_q1 + c0, dd);
      tc::tmem_wait_ld();
      if (row) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int col = c0 + i;
          const float val = ntl > 0 ? __uint_as_float(dd[i]) : 0.f;
          if (col < width) dst[t * (width + 1) + col] = val;
          else if (col == width) dst[t * (width + 1) + width] = val;
        }
      }
    }
    if (part == 1) {
      uint32_t dd[16];
      tc::tmem_ld16(arow + e.col_q2, dd);
      tc::tmem_wait_ld();
      if (row) {
        float *d2 = dst + hidden * (width + 1);
#pragma unroll
        for (int o = 0; o < kMaxOut; ++o)
          if (o < out_ch) d2[o * (hidden + 1) + t] = ntl > 0 ? __uint_as_float(dd[o]) : 0.f;
      }
    }
    if (part == 2 && q == 0 && lane < out_ch) {
      float *d2 = dst + hidden * (width + 1);
      d2[lane * (hidden + 1) + hidden] = dq2s[lane];
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
cudaError_t launch_proj_bwd_t(const Launch &L, const Geom &g, const ProjArgs &a, const void *v,
                              const void *du, void *dv, float *partial, int *nparts) {
  using K = QKind<T>;
  const PbGeom e = pb_geom(a.width, a.out_ch);
  CUtensorMap tmv, tmdu;
  memset(&tmv, 0, sizeof(tmv));
  memset(&tmdu, 0, sizeof(tmdu));
  const uint64_t rowb = (uint64_t)g.N * 2;
  {
    const uint64_t dims[4] = {(uint64_t)g.N, 1u, (uint64_t)a.width, (uint64_t)g.B};
    const uint64_t str[3] = {rowb, rowb, rowb * (uint64_t)a.width};
    const uint32_t box[4] = {(uint32_t)PB_XBOX, 1u, (uint32_t)a.width, 1u};
    if (!encode_tmap_4d(&tmv, K::tmap, v, dims, str, box, true)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[4] = {(uint64_t)g.N, 1u, (uint64_t)a.out_ch, (uint64_t)g.B};
    const uint64_t str[3] = {rowb, rowb, rowb * (uint64_t)a.out_ch};
    const uint32_t box[4] = {(uint32_t)ROWS, 1u, (uint32_t)a.out_ch, 1u};
    if (!encode_tmap_4d(&tmdu, K::tmap, du, dims, str, box)) return cudaErrorInvalidValue;
  }
  const long long ntiles = g.B * (g.N / ROWS);
  const int grid = (int)(ntiles < L.num_sms ? ntiles : L.num_sms);
  *nparts = grid;
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)e.total);
    kern<<<grid, THREADS, e.total, L.stream>>>(tmv, tmdu, a, dv, partial);
  };
  if (a.width <= 16) go(k_proj_bwd_pipe<T, 16>);
  else if (a.width <= 32) go(k_proj_bwd_pipe<T, 32>);
  else go(k_proj_bwd_pipe<T, 64>);
  return cudaGetLastError();
}

}  // namespace

bool proj_pipe_supported(const Geom &g, int dtype, int width, int hidden, int out_ch,
                         const void *v) {
  if (g.N % ROWS != 0 || g.N > (1LL << 30) || g.B > (1LL << 30)) return false;
  if (out_ch > kMaxOut || width > 64 || hidden < 1) return false;
  if ((reinterpret_cast<uintptr_t>(v) & 15) != 0) return false;
  const bool tf32 = dtype == DT_F32;
  const ProjGeom e = proj_geom(width, hidden, tf32 ? 4 : 2, tf32);
  if (e.HP > 256 || e.used > 512) return false;
  return e.NS >= 2 && e.total <= kSmemMax;
}

cudaError_t launch_proj_pipe(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                             int out_ch, const void *v, const void *Q1, const void *q1,
                             const void *Q2, const void *q2, void *u) {
  ProjArgs a{};
  a.Q1 = Q1;
  a.q1 = q1;
  a.Q2 = Q2;
  a.q2 = q2;
  a.u = u;
  a.err = L.err;
  a.B = g.B;
  a.N = g.N;
  a.width = width;
  a.hidden = hidden;
  a.out_ch = out_ch;
  launch_begin(L);
  cudaError_t err = dtype == DT_F32   ? launch_t<float>(L, g, a, v)
                    : dtype == DT_F16 ? launch_t<__half>(L, g, a, v)
                                      : launch_t<__nv_bfloat16>(L, g, a, v);
  launch_end(L, "proj_fwd_pipe");
  return err;
}


bool proj_bwd_pipe_supported(const Geom &g, int dtype, int width, int hidden, int out_ch,
                             const void *v, const void *du, const void *dv) {
  if (dtype == DT_F32) return false;
  if (g.N % ROWS != 0 || g.N > (1LL << 30) || g.B > (1LL << 30)) return false;
  if (width % 16 != 0 || width > 64 || hidden < 1 || hidden > ROWS) return false;
  if (out_ch < 1 || out_ch > kMaxOut) return false;
  if (((reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(du) |
        reinterpret_cast<uintptr_t>(dv)) & 15) != 0)
    return false;
  const PbGeom e = pb_geom(width, out_ch);
  return e.used <= 512 && e.NS >= 2 && e.total <= kSmemMax;
}

cudaError_t launch_proj_bwd_pipe(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                                 int out_ch, const void *v, const void *du, const void *Q1,
                                 const void *q1, const void *Q2, void *dv, float *partial,
                                 int *nparts) {
  ProjArgs a{};
  a.Q1 = Q1;
  a.q1 = q1;
  a.Q2 = Q2;
  a.err = L.err;
  a.B = g.B;
  a.N = g.N;
  a.width = width;
  a.hidden = hidden;
  a.out_ch = out_ch;
  launch_begin(L);
  cudaError_t err = dtype == DT_F16
                        ? launch_proj_bwd_t<__half>(L, g, a, v, du, dv, partial, nparts)
                        : launch_proj_bwd_t<__nv_bfloat16>(L, g, a, v, du, dv, partial, nparts);
  launch_end(L, "proj_bwd_pipe");
  return err;
}

}  // namespace fno
