// Per-mode complex channel mixing (step S3) on the tensor cores, for bfloat16
// weights and 64 output channels: the forward yhat = w_k R^T xhat and the
// input adjoint dxhat = w_k conj(R) D as one real GEMM per mode.
//
// For a mode k, write the complex reduction  Y[b, n] = sum_r X[b, r] A_k(n, r)
// in real form: with K index 2 r + c' (c' = 0 real, 1 imaginary part of X)
// and row index 2 n + c (c = 0 real, 1 imaginary part of Y),
//     D[2n + c, b] = sum_{r, c'} Ablk[2n + c, 2r + c'] X[b, 2r + c']
// where each 2 x 2 block of Ablk is the real matrix of multiplication by
//     forward:  A(n, r) = R[r, n]         ( Rr  -Ri )   rows 2n, 2n + 1
//                                        ( Ri   Rr )
//     adjoint:  A(n, r) = conj R[n, r]    ( Rr   Ri )
//                                        (-Ri   Rr )
// M = 2 x 64 = 128 rows (TMEM lanes), N = the batch (padded to a multiple of
// 16 with zero rows), K = 2 x (reduced channels).  The weights are bfloat16
// and enter exactly; X (float32 spectra) enters as a bfloat16 pair hi + lo
// (hi = X rounded, lo = X - hi rounded), two MMA chains into one fp32
// accumulator, so the products keep about 16 mantissa bits of X.
//
// One CTA per MB (4 or 2) consecutive modes, K a multiple of 4: all threads
// gather the modes' operands from global memory into shared memory in the
// tcgen05 K-major core-matrix layout (R as one load of the MB modes' (re, im)
// pairs per (i, o), X as 16-byte loads of the MB modes), one elected thread
// issues the chains, every thread waits on the commit (bounded), and the
// sixteen warps read the accumulators back: warp w takes TMEM lane quarter
// w % 4 (32 rows = 16 output channels, real and imaginary in neighbouring
// lanes) and every fourth 8-column chunk of the batch; each thread writes, per
// batch entry, the MB modes of one output channel as one contiguous run,
// scaled by the inverse transform's c_k / N.  Sixteen warps and one pass of
// loads per thread keep the gather's memory latency to about one round trip
// (eight warps and three passes left the kernel waiting on loads).
#include "fno_common.cuh"
#include "fno_kernels.cuh"
#include "tc_util.cuh"
#include "tma_util.cuh"

namespace fno {

namespace {

constexpr int MT_THREADS = 512;
constexpr int MT_RB = 8, MT_XB = 4;          // weight / spectrum loads per thread and pass
constexpr int MT_ROWS = 128;                 // 2 x 64 output channels
constexpr size_t MT_SMEM_MAX = 227 * 1024;

struct MtGeom {
  int NB;            // batch padded to a multiple of 16 (the MMA's N)
  uint32_t sbo;      // bytes between 8-row groups (K = 2 NR bf16 per row)
  size_t a_bytes, b_bytes, a0, b0, bar, tslot, total;
  uint32_t cols;     // TMEM columns allocated (power of two >= MB NB)
};

__host__ __device__ inline MtGeom mt_geom(long long B, int NR, int MB) {
  MtGeom e;
  e.NB = (int)((B + 15) / 16 * 16);
  e.sbo = (uint32_t)(2 * NR * 2 / 16) * 128u;
  e.a_bytes = (size_t)MT_ROWS * 2 * NR * 2;
  e.b_bytes = (size_t)e.NB * 2 * NR * 2;
  e.a0 = 0;
  e.b0 = e.a0 + (size_t)MB * e.a_bytes;
  e.bar = e.b0 + (size_t)MB * 2 * e.b_bytes;
  e.tslot = e.bar + 8;
  e.total = e.tslot + 8;
  uint32_t c = 32;
  while (c < (uint32_t)(MB * e.NB)) c *= 2;
  e.cols = c;
  return e;
}

// byte offset of element (row, kel) of a K-major no-swizzle bf16 operand
__device__ __forceinline__ uint32_t mt_off(int row, int kel, uint32_t sbo) {
  const int kb = kel * 2;
  return (uint32_t)(row >> 3) * sbo + (uint32_t)(kb >> 4) * 128u + (uint32_t)(row & 7) * 16u +
         (uint32_t)(kb & 15);
}

__device__ __forceinline__ uint32_t bf16_bits(float x) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// X value -> (hi, lo) bfloat16 pairs packed as (re | im << 16)
__device__ __forceinline__ void split_pair(float2 v, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat16 hr = __float2bfloat16_rn(v.x), hi_ = __float2bfloat16_rn(v.y);
  hi = (uint32_t)__bfloat16_as_ushort(hr) | ((uint32_t)__bfloat16_as_ushort(hi_) << 16);
  lo = bf16_bits(v.x - __bfloat162float(hr)) | (bf16_bits(v.y - __bfloat162float(hi_)) << 16);
}

// X [B][NR][K] float2, R [Ci][Co][K] (re, im) bfloat16, Y [B][64][K] float2;
// NR = Ci (forward) or Co (adjoint); the other channel count is 64.
template <int MB, bool ADJ>
__global__ void __launch_bounds__(MT_THREADS, 1)
    k_mix_tc(const float2 *__restrict__ X, const __nv_bfloat16 *__restrict__ R,
             float2 *__restrict__ Y, int B, int Ci, int Co, long long K, int mL, int NL,
             float inv_n, int *err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int NR = ADJ ? Co : Ci;
  const MtGeom e = mt_geom(B, NR, MB);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + e.bar);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + e.tslot);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long k0 = (long long)blockIdx.x * MB;

  if (warp == 0) {
    tc::tmem_alloc(tslot, e.cols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tma::fence_barrier_init();
  }

  // ---- operands.  Weights: pair p -> (n, r) with the low bits on (n & 3,
  // r & 3), so that a warp's four-byte stores fall in 16 banks of a core-matrix
  // row set.  Spectra: pair p -> (b, r) with the low bits on (b & 7, r & 3);
  // rows b >= B are zero.  Each pass issues MT_RB weight loads and MT_XB
  // spectrum loads per thread before any store, so one pass waits out one
  // memory latency.
  {
    const int nq = 64 / 4;                       // n groups of four
    const int nrp = 64 * NR;                     // weight pairs
    const int nbq = e.NB / 8;
    const int nxp = e.NB * NR;                   // spectrum pairs
    for (int it = 0; it * MT_RB * MT_THREADS < nrp || it * MT_XB * MT_THREADS < nxp; ++it) {
      uint4 rv[MT_RB];
      int nn[MT_RB], rr[MT_RB];
#pragma unroll
      for (int u = 0; u < MT_RB; ++u) {
        const int p = (it * MT_RB + u) * MT_THREADS + tid;
        const int q = p >> 4;
        nn[u] = (q % nq) * 4 + (p & 3);
        rr[u] = (q / nq) * 4 + ((p >> 2) & 3);
        rv[u] = make_uint4(0u, 0u, 0u, 0u);
        if (p < nrp) {
          const int i = ADJ ? nn[u] : rr[u], o = ADJ ? rr[u] : nn[u];
          const __nv_bfloat16 *src = R + 2 * (((long long)i * Co + o) * K + k0);
          if constexpr (MB == 4) {
            rv[u] = __ldg(reinterpret_cast<const uint4 *>(src));
          } else {
            const uint2 t = __ldg(reinterpret_cast<const uint2 *>(src));
            rv[u].x = t.x;
            rv[u].y = t.y;
          }
        }
      }
      float4 xv[MT_XB][2];
      int bb[MT_XB], xr[MT_XB];
#pragma unroll
      for (int u = 0; u < MT_XB; ++u) {
        const int p = (it * MT_XB + u) * MT_THREADS + tid;
        const int q = p >> 5;
        bb[u] = (q % nbq) * 8 + (p & 7);
        xr[u] = (q / nbq) * 4 + ((p >> 3) & 3);
        xv[u][0] = xv[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p < nxp && bb[u] < B) {
          const float4 *src =
              reinterpret_cast<const float4 *>(X + ((long long)bb[u] * NR + xr[u]) * K + k0);
          xv[u][0] = __ldg(src);
          if constexpr (MB == 4) xv[u][1] = __ldg(src + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < MT_RB; ++u) {
        if ((it * MT_RB + u) * MT_THREADS + tid >= nrp) break;
        const uint32_t w4[4] = {rv[u].x, rv[u].y, rv[u].z, rv[u].w};   // (re | im << 16) per mode
        const uint32_t o0 = mt_off(2 * nn[u], 2 * rr[u], e.sbo);
        const uint32_t o1 = mt_off(2 * nn[u] + 1, 2 * rr[u], e.sbo);
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          const uint32_t re = w4[m] & 0xFFFFu, im = w4[m] >> 16;
          const uint32_t nim = im ^ 0x8000u;
          // forward rows (Rr, -Ri) / (Ri, Rr); adjoint rows (Rr, Ri) / (-Ri, Rr)
          const uint32_t row0 = ADJ ? (re | (im << 16)) : (re | (nim << 16));
          const uint32_t row1 = ADJ ? (nim | (re << 16)) : (im | (re << 16));
          unsigned char *am = smem + e.a0 + (size_t)m * e.a_bytes;
          *reinterpret_cast<uint32_t *>(am + o0) = row0;
          *reinterpret_cast<uint32_t *>(am + o1) = row1;
        }
      }
#pragma unroll
      for (int u = 0; u < MT_XB; ++u) {
        if ((it * MT_XB + u) * MT_THREADS + tid >= nxp) break;
        const float2 v4[4] = {make_float2(xv[u][0].x, xv[u][0].y), make_float2(xv[u][0].z, xv[u][0].w),
                              make_float2(xv[u][1].x, xv[u][1].y), make_float2(xv[u][1].z, xv[u][1].w)};
        const uint32_t off = mt_off(bb[u], 2 * xr[u], e.sbo);
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          uint32_t hi, lo;
          split_pair(v4[m], hi, lo);
          unsigned char *bm = smem + e.b0 + (size_t)(2 * m) * e.b_bytes;
          *reinterpret_cast<uint32_t *>(bm + off) = hi;
          *reinterpret_cast<uint32_t *>(bm + e.b_bytes + off) = lo;
        }
      }
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tslot;

  // ---- MMA: per mode, the hi chain then the lo chain into D_m
  if (warp == 0) {
    if (tc::elect_one()) {
      const uint32_t idesc = tc::instr_desc(tc::FMT_BF16, MT_ROWS, e.NB);
      const int nks = 2 * NR / 16;
      for (int m = 0; m < MB; ++m) {
        const uint32_t d = tbase + (uint32_t)(m * e.NB);
        const uint64_t ad = tc::smem_desc_kmajor(tc::smem_u32(smem + e.a0 + (size_t)m * e.a_bytes),
                                                 128, e.sbo);
        const uint64_t bh = tc::smem_desc_kmajor(
            tc::smem_u32(smem + e.b0 + (size_t)(2 * m) * e.b_bytes), 128, e.sbo);
        const uint64_t bl = tc::smem_desc_kmajor(
            tc::smem_u32(smem + e.b0 + (size_t)(2 * m + 1) * e.b_bytes), 128, e.sbo);
        for (int ks = 0; ks < nks; ++ks)
          tc::mma_f16_ss(d, ad + 16u * ks, bh + 16u * ks, idesc, ks > 0 ? 1u : 0u);
        for (int ks = 0; ks < nks; ++ks) tc::mma_f16_ss(d, ad + 16u * ks, bl + 16u * ks, idesc, 1u);
      }
      tc::mma_commit(bar);
    }
    __syncwarp();
  }
  bool ok = tc::mbar_wait(bar, 0, err);
  if (!ok) tc::mbar_wait(bar, 0, nullptr);   // drain before TMEM is released
  tc::fence_after_sync();

  // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. (16 output channels,
  // real and imaginary parts in neighbouring lanes) and the 8-column batch
  // chunks w / 4, w / 4 + 4, ...
  if (ok) {
    const int q = warp & 3;
    const int row = 32 * q + lane;               // 2 n + c
    const int n = row >> 1, c = row & 1;
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    float wk[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) wk[m] = mode_weight((int)((k0 + m) % mL), NL, inv_n);
    for (int c0 = (warp >> 2) * 8; c0 < e.NB; c0 += (MT_THREADS / 128) * 8) {
      uint32_t v[MB][8];
#pragma unroll
      for (int m = 0; m < MB; ++m) tc::tmem_ld8(lane_base + (uint32_t)(m * e.NB + c0), v[m]);
      tc::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float own[MB], oth[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          own[m] = __uint_as_float(v[m][j]);
          oth[m] = __shfl_xor_sync(0xffffffffu, own[m], 1);
        }
        const int b = c0 + j;
        // the real-part lane stores even j, the imaginary-part lane odd j
        if ((j & 1) == c && b < B) {
          float2 y[MB];
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            const float re = c == 0 ? own[m] : oth[m], im = c == 0 ? oth[m] : own[m];
            y[m] = make_float2(wk[m] * re, wk[m] * im);
          }
          float4 *dst = reinterpret_cast<float4 *>(Y + ((long long)b * 64 + n) * K + k0);
          dst[0] = make_float4(y[0].x, y[0].y, y[1].x, y[1].y);
          if constexpr (MB == 4) dst[1] = make_float4(y[2].x, y[2].y, y[3].x, y[3].y);
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

// ---------------------------------------------------------------------------
// dR[i, o, k] = w_k sum_b conj(xhat[b, i, k]) D[b, o, k] for 64 input channels:
// per mode the real GEMM, rows 2 i + c (c = 0 real, 1 imaginary part of dR),
// columns o, K index 2 b + c',
//     D_acc[2i + c, o] = sum_{b, c'} Ablk[2i + c, 2b + c'] Dv[o, 2b + c']
//     rows 2i: (Xr, Xi)    rows 2i + 1: (-Xi, Xr)    Dv[o, 2b..2b+1] = (Dr, Di)
// M = 128, N = Co padded to 16, K = 2 x batch padded to 8.  Both operands are
// float32 spectra and enter as bfloat16 pairs hi + lo, in three chains
// (A_hi B_hi, A_hi B_lo, A_lo B_hi) into one fp32 accumulator: about 16
// mantissa bits per product, for 16-bit storage.  The gather, issue, bounded
// wait and read-back follow k_mix_tc; the read-back writes, per (i, o), the MB
// modes of dR contiguously.
struct DrGeom {
  int KB, NP;        // batch padded to 8, output channels padded to 16
  uint32_t sbo;
  size_t a_bytes, b_bytes, a0, b0, bar, tslot, total;
  uint32_t cols;
};

__host__ __device__ inline DrGeom dr_geom(long long B, int Co, int MB) {
  DrGeom e;
  e.KB = (int)((B + 7) / 8 * 8);
  e.NP = (Co + 15) / 16 * 16;
  const int kel = 2 * e.KB;
  e.sbo = (uint32_t)(kel * 2 / 16) * 128u;
  e.a_bytes = (size_t)MT_ROWS * kel * 2;     // one of A_hi, A_lo
  e.b_bytes = (size_t)e.NP * kel * 2;        // one of B_hi, B_lo
  e.a0 = 0;
  e.b0 = (size_t)MB * 2 * e.a_bytes;
  e.bar = e.b0 + (size_t)MB * 2 * e.b_bytes;
  e.tslot = e.bar + 8;
  e.total = e.tslot + 8;
  uint32_t c = 32;
  while (c < (uint32_t)(MB * e.NP)) c *= 2;
  e.cols = c;
  return e;
}

__device__ __forceinline__ uint32_t neg_bf16_lo(uint32_t w) { return w ^ 0x8000u; }

template <int MB>
__global__ void __launch_bounds__(MT_THREADS, 1)
    k_mix_tc_dr(const float2 *__restrict__ X, const float2 *__restrict__ Dsp,
                float *__restrict__ dR, int B, int Co, long long K, int mL, int NL, float inv_n,
                int *err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  constexpr int Ci = 64;
  const DrGeom e = dr_geom(B, Co, MB);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + e.bar);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + e.tslot);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long k0 = (long long)blockIdx.x * MB;

  if (warp == 0) {
    tc::tmem_alloc(tslot, e.cols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tma::fence_barrier_init();
  }
  // ---- operands, one pass of loads per thread before the stores.  A from
  // xhat: pair p -> (i, b) with the low bits on (i & 3, b & 3); B from D: pair
  // p -> (o, b) with the low bits on (o & 7, b & 3); padded rows are zero.
  {
    const int nxp = 64 * e.KB, nq8 = e.NP / 8, ndp = e.NP * e.KB;
    for (int it = 0; it * MT_XB * MT_THREADS < nxp || it * MT_XB * MT_THREADS < ndp; ++it) {
      float4 xv[MT_XB][2], dv[MT_XB][2];
      int xi_[MT_XB], xb_[MT_XB], dor[MT_XB], db_[MT_XB];
#pragma unroll
      for (int u = 0; u < MT_XB; ++u) {
        const int p = (it * MT_XB + u) * MT_THREADS + tid;
        const int q = p >> 4;
        xi_[u] = (q % 16) * 4 + (p & 3);
        xb_[u] = (q / 16) * 4 + ((p >> 2) & 3);
        xv[u][0] = xv[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p < nxp && xb_[u] < B) {
          const float4 *src =
              reinterpret_cast<const float4 *>(X + ((long long)xb_[u] * Ci + xi_[u]) * K + k0);
          xv[u][0] = __ldg(src);
          if constexpr (MB == 4) xv[u][1] = __ldg(src + 1);
        }
        const int q2 = p >> 5;
        dor[u] = (q2 % nq8) * 8 + (p & 7);
        db_[u] = (q2 / nq8) * 4 + ((p >> 3) & 3);
        dv[u][0] = dv[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p < ndp && db_[u] < B && dor[u] < Co) {
          const float4 *src =
              reinterpret_cast<const float4 *>(Dsp + ((long long)db_[u] * Co + dor[u]) * K + k0);
          dv[u][0] = __ldg(src);
          if constexpr (MB == 4) dv[u][1] = __ldg(src + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < MT_XB; ++u) {
        if ((it * MT_XB + u) * MT_THREADS + tid < nxp) {
          const float2 v4[4] = {make_float2(xv[u][0].x, xv[u][0].y), make_float2(xv[u][0].z, xv[u][0].w),
                                make_float2(xv[u][1].x, xv[u][1].y), make_float2(xv[u][1].z, xv[u][1].w)};
          const uint32_t o0 = mt_off(2 * xi_[u], 2 * xb_[u], e.sbo);
          const uint32_t o1 = mt_off(2 * xi_[u] + 1, 2 * xb_[u], e.sbo);
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            uint32_t hi, lo;                       // (re | im << 16)
            split_pair(v4[m], hi, lo);
            unsigned char *ah = smem + e.a0 + (size_t)(2 * m) * e.a_bytes;
            unsigned char *al = ah + e.a_bytes;
            // row 2i: (Xr, Xi); row 2i + 1: (-Xi, Xr)
            *reinterpret_cast<uint32_t *>(ah + o0) = hi;
            *reinterpret_cast<uint32_t *>(al + o0) = lo;
            *reinterpret_cast<uint32_t *>(ah + o1) = neg_bf16_lo(hi >> 16) | (hi << 16);
            *reinterpret_cast<uint32_t *>(al + o1) = neg_bf16_lo(lo >> 16) | (lo << 16);
          }
        }
        if ((it * MT_XB + u) * MT_THREADS + tid < ndp) {
          const float2 v4[4] = {make_float2(dv[u][0].x, dv[u][0].y), make_float2(dv[u][0].z, dv[u][0].w),
                                make_float2(dv[u][1].x, dv[u][1].y), make_float2(dv[u][1].z, dv[u][1].w)};
          const uint32_t off = mt_off(dor[u], 2 * db_[u], e.sbo);
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            uint32_t hi, lo;
            split_pair(v4[m], hi, lo);
            unsigned char *bh = smem + e.b0 + (size_t)(2 * m) * e.b_bytes;
            *reinterpret_cast<uint32_t *>(bh + off) = hi;
            *reinterpret_cast<uint32_t *>(bh + e.b_bytes + off) = lo;
          }
        }
      }
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tslot;

  if (warp == 0) {
    if (tc::elect_one()) {
      const uint32_t idesc = tc::instr_desc(tc::FMT_BF16, MT_ROWS, e.NP);
      const int nks = 2 * e.KB / 16;
      for (int m = 0; m < MB; ++m) {
        const uint32_t d = tbase + (uint32_t)(m * e.NP);
        unsigned char *am = smem + e.a0 + (size_t)(2 * m) * e.a_bytes;
        unsigned char *bm = smem + e.b0 + (size_t)(2 * m) * e.b_bytes;
        const uint64_t ah = tc::smem_desc_kmajor(tc::smem_u32(am), 128, e.sbo);
        const uint64_t al = tc::smem_desc_kmajor(tc::smem_u32(am + e.a_bytes), 128, e.sbo);
        const uint64_t bh = tc::smem_desc_kmajor(tc::smem_u32(bm), 128, e.sbo);
        const uint64_t bl = tc::smem_desc_kmajor(tc::smem_u32(bm + e.b_bytes), 128, e.sbo);
        for (int ks = 0; ks < nks; ++ks)
          tc::mma_f16_ss(d, ah + 16u * ks, bh + 16u * ks, idesc, ks > 0 ? 1u : 0u);
        for (int ks = 0; ks < nks; ++ks) tc::mma_f16_ss(d, ah + 16u * ks, bl + 16u * ks, idesc, 1u);
        for (int ks = 0; ks < nks; ++ks) tc::mma_f16_ss(d, al + 16u * ks, bh + 16u * ks, idesc, 1u);
      }
      tc::mma_commit(bar);
    }
    __syncwarp();
  }
  bool ok = tc::mbar_wait(bar, 0, err);
  if (!ok) tc::mbar_wait(bar, 0, nullptr);   // drain before TMEM is released
  tc::fence_after_sync();

  if (ok) {
    const int q = warp & 3;
    const int row = 32 * q + lane;               // 2 i + c
    const int i = row >> 1, c = row & 1;
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    float wk[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) wk[m] = mode_weight((int)((k0 + m) % mL), NL, inv_n);
    for (int c0 = (warp >> 2) * 8; c0 < e.NP; c0 += (MT_THREADS / 128) * 8) {
      uint32_t v[MB][8];
#pragma unroll
      for (int m = 0; m < MB; ++m) tc::tmem_ld8(lane_base + (uint32_t)(m * e.NP + c0), v[m]);
      tc::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float own[MB], oth[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          own[m] = __uint_as_float(v[m][j]);
          oth[m] = __shfl_xor_sync(0xffffffffu, own[m], 1);
        }
        const int o = c0 + j;
        if ((j & 1) == c && o < Co) {
          float2 y[MB];
#pragma unroll
          for (int m = 0; m < MB; ++m) {
            const float re = c == 0 ? own[m] : oth[m], im = c == 0 ? oth[m] : own[m];
            y[m] = make_float2(wk[m] * re, wk[m] * im);
          }
          float4 *dst = reinterpret_cast<float4 *>(dR + 2 * (((long long)i * Co + o) * K + k0));
          dst[0] = make_float4(y[0].x, y[0].y, y[1].x, y[1].y);
          if constexpr (MB == 4) dst[1] = make_float4(y[2].x, y[2].y, y[3].x, y[3].y);
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

inline int dr_modes(long long B, int Co) {
  if (dr_geom(B, Co, 4).total <= MT_SMEM_MAX) return 4;
  if (dr_geom(B, Co, 2).total <= MT_SMEM_MAX) return 2;
  return 0;
}

inline int mt_modes(long long B, int NR) {
  if (mt_geom(B, NR, 4).total <= MT_SMEM_MAX) return 4;
  if (mt_geom(B, NR, 2).total <= MT_SMEM_MAX) return 2;
  return 0;
}

}  // namespace

bool mix_tc_supported(const Geom &g, int dtype, bool adj, int Ci, int Co, const void *X,
                      const void *R, const void *Y) {
  const int NR = adj ? Co : Ci, NOUT = adj ? Ci : Co;
  if (dtype != DT_BF16 || NOUT != 64) return false;
  if (NR % 8 != 0 || NR > 64 || g.B < 1 || g.B > 64) return false;
  if (g.K % 4 != 0) return false;   // 16-byte loads of four modes from aligned rows
  if (((uintptr_t)X | (uintptr_t)R | (uintptr_t)Y) & 31) return false;
  return mt_modes(g.B, NR) > 0;
}

cudaError_t launch_mix_tc(const Launch &L, const Geom &g, bool adj, int Ci, int Co,
                          const float2 *X, const void *R, float2 *Y) {
  const int NR = adj ? Co : Ci;
  const int mb = mt_modes(g.B, NR);
  const MtGeom e = mt_geom(g.B, NR, mb);
  const unsigned grid = (unsigned)((g.K + mb - 1) / mb);
  auto go = [&](auto kern) {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)e.total);
    if (r != cudaSuccess) return r;
    kern<<<grid, MT_THREADS, e.total, L.stream>>>(X, (const __nv_bfloat16 *)R, Y, (int)g.B, Ci,
                                                   Co, g.K, g.mL, g.NL, g.inv_n, L.err);
    return cudaGetLastError();
  };
  if (adj) return mb == 4 ? go(k_mix_tc<4, true>) : go(k_mix_tc<2, true>);
  return mb == 4 ? go(k_mix_tc<4, false>) : go(k_mix_tc<2, false>);
}

}  // namespace fno

namespace fno {

bool mix_tc_dr_supported(const Geom &g, int dtype, int Ci, int Co, const void *X, const void *D,
                         const void *dR) {
  if (dtype == DT_F32 || Ci != 64 || Co < 1 || Co > 64) return false;
  if (g.B < 1 || g.B > 64 || g.K % 4 != 0) return false;
  if (((uintptr_t)X | (uintptr_t)D | (uintptr_t)dR) & 31) return false;
  return dr_modes(g.B, Co) > 0;
}

cudaError_t launch_mix_tc_dr(const Launch &L, const Geom &g, int Co, const float2 *X,
                             const float2 *D, float *dR) {
  const int mb = dr_modes(g.B, Co);
  const DrGeom e = dr_geom(g.B, Co, mb);
  const unsigned grid = (unsigned)((g.K + mb - 1) / mb);
  auto go = [&](auto kern) {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)e.total);
    if (r != cudaSuccess) return r;
    kern<<<grid, MT_THREADS, e.total, L.stream>>>(X, D, dR, (int)g.B, Co, g.K, g.mL, g.NL,
                                                   g.inv_n, L.err);
    return cudaGetLastError();
  };
  return mb == 4 ? go(k_mix_tc_dr<4>) : go(k_mix_tc_dr<2>);
}

}  // namespace fno
