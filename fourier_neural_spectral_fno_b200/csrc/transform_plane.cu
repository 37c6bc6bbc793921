// Truncated forward transform (steps S0-S2), whole planes per CTA: the
// HBM-streaming form of the pruned radix-16 FFT of transform_fft.cu.
//
// One persistent CTA per SM walks the (sample, channel[, outer]) planes.  A
// producer warp streams the plane's rows into a shared-memory ring with a few
// untiled bulk async copies per batch of rows (one per group of 15 consecutive
// rows; measured, a copy per row left the consumers waiting a third of the
// time on the copy engine), signalled through mbarrier transaction counts;
// fifteen consumer warps turn each batch of rows
// into last-axis spectra (the pruned FFT of transform_fft.cu: one register
// FFT16 of a packed pair of real subsequences per thread, the real-pair
// combine, a shuffle reduce-scatter over the row's threads) and keep them in
// shared memory, so the ring is refilled while they compute.
//
// With the whole plane's row spectra X1[n, k] on chip, the slab axis is a
// pruned radix-16 FFT as well (S = 16 Qs, n = Qs a + r):
//   X2[q, k] = sum_r exp(-2 pi i kq r / S) Z_r[kq mod 16, k],
//   Z_r[p, k] = sum_a X1[Qs a + r, k] exp(-2 pi i p a / 16),
// first the Qs x m FFT16s in place (each owns the rows r mod Qs of one
// column), then the twiddled sums over r for the kept kq only.  The plane's
// spectrum is written once; x is read from HBM exactly once.
#include "fft16.cuh"
#include "fno_common.cuh"
#include "fno_kernels.cuh"
#include "tc_util.cuh"
#include "tma_util.cuh"

namespace fno {

namespace {

// fifteen consumer warps + the producer = 16 warps, four per sub-partition,
// which leaves each thread 128 registers
constexpr int PL_CONSUMERS = 480;
constexpr int PL_THREADS = PL_CONSUMERS + 32;   // + the producer warp
constexpr int PL_MAXSTAGES = 4;
constexpr size_t PL_SMEM_MAX = 227 * 1024;

// A batch of RB = 15 G rows (G = rows per consumer warp) sits in G groups of 15
// consecutive rows, one bulk copy each; warp w takes the rows w, w + 15, ...,
// one per group, and the groups are GS = 15 RS + PADG bytes apart, PADG being
// the bytes a row's threads read at once, so a warp's rows lie on successive
// banks and its loads take the minimal number of wavefronts.
constexpr int PL_WARPS = PL_CONSUMERS / 32;   // rows per group

struct PlaneGeom {
  int T, RB, G, MP, Qs, NS, nin, RS;
  size_t GS, stage, x1, twc, tw2, bar, total;
};

// modes padded so that the 2T threads of a row split them evenly
__host__ __device__ inline int pl_mp(int mL, int T) {
  const int m = mL <= 8 ? 8 : mL <= 16 ? 16 : mL <= 24 ? 24 : 32;
  return (T == 8 && m % 16) ? m + 8 : m;
}
__host__ __device__ inline size_t pl_al(size_t v, size_t a) { return (v + a - 1) / a * a; }

// es: storage element bytes; nin: input arrays streamed (2 for dz = dy GELU'(pre))
__host__ __device__ inline PlaneGeom plane_geom(int S, int NL, int mL, int QS, int es, int nin) {
  PlaneGeom p{};
  p.T = NL / 64;
  p.RB = PL_CONSUMERS / (2 * p.T);
  p.G = 32 / (2 * p.T);
  p.MP = pl_mp(mL, p.T);
  p.Qs = S / 16;
  p.nin = nin;
  p.RS = NL * es;                                  // rows dense within a group
  p.GS = pl_al((size_t)PL_WARPS * p.RS + (size_t)(2 * p.T) * 2 * es, 16);   // copy alignment
  p.stage = pl_al((size_t)nin * p.G * p.GS, 128);
  const size_t x1 = sizeof(float2) * (size_t)S * (p.MP + 1);
  const size_t twc = sizeof(float2) * 4 * (size_t)p.MP * p.T;
  const size_t tw2 = sizeof(float2) * (size_t)QS * p.Qs;
  const size_t bar = sizeof(uint64_t) * 2 * PL_MAXSTAGES;
  const size_t fixed = x1 + twc + tw2 + bar + 128;
  const size_t room = PL_SMEM_MAX > fixed ? PL_SMEM_MAX - fixed : 0;
  const size_t ns = room / p.stage;
  p.NS = (int)(ns < (size_t)PL_MAXSTAGES ? ns : (size_t)PL_MAXSTAGES);
  size_t off = (size_t)(p.NS > 0 ? p.NS : 0) * p.stage;
  p.x1 = off; off += x1;
  p.twc = off; off += twc;
  p.tw2 = off; off += tw2;
  p.bar = pl_al(off, 8); off = p.bar + bar;
  p.total = off;
  return p;
}

struct PlaneArgs {
  const void *in0, *in1;   // [planes][S][NL] (in1: pre, for dz)
  float2 *out;             // [planes][QS][mL]
  long long planes;
  int S, NL, mL, mS, QS, tanh_in;
  int *err;
};

// two consecutive storage elements as floats
__device__ __forceinline__ float2 ld_pair(const float *p) {
  return *reinterpret_cast<const float2 *>(p);
}
__device__ __forceinline__ float2 ld_pair(const __half *p) {
  return __half22float2(*reinterpret_cast<const __half2 *>(p));
}
__device__ __forceinline__ float2 ld_pair(const __nv_bfloat16 *p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(PL_CONSUMERS) : "memory");
}

// acc[k] += Z[m] alpha + conj(Z[-m]) beta (m = k mod 16): the twiddled sum of
// two real subsequences packed as one complex FFT16 (see transform_fft.cu)
template <int MP>
__device__ __forceinline__ void combine_pair(float2 (&acc)[MP], const float2 (&Z)[16],
                                             const float2 *tw, int T2) {
#pragma unroll
  for (int k = 0; k < MP; ++k) {
    const int m = k & 15, mm = (16 - m) & 15;
    const float4 ab = *reinterpret_cast<const float4 *>(tw + (size_t)k * T2 * 2);
    const float2 z = Z[m], w = Z[mm];
    acc[k].x = fmaf(z.x, ab.x, fmaf(-z.y, ab.y, fmaf(w.x, ab.z, fmaf(w.y, ab.w, acc[k].x))));
    acc[k].y = fmaf(z.x, ab.y, fmaf(z.y, ab.x, fmaf(w.x, ab.w, fmaf(-w.y, ab.z, acc[k].y))));
  }
}

// reduce-scatter of MP values over T consecutive lanes (lane j keeps
// k in [j MP/T, (j+1) MP/T) in v[0..MP/T))
template <int MP, int T>
__device__ __forceinline__ void rs_lanes(float2 (&v)[MP], int j) {
  int cnt = MP;
#pragma unroll
  for (int d = T / 2; d >= 1; d /= 2) {
    const bool upper = (j & d) != 0;
    cnt /= 2;
#pragma unroll
    for (int i = 0; i < MP / 2; ++i) {
      if (i < cnt) {
        const float2 keep = upper ? v[i + cnt] : v[i];
        const float2 send = upper ? v[i] : v[i + cnt];
        const float rx = __shfl_xor_sync(0xffffffffu, send.x, d);
        const float ry = __shfl_xor_sync(0xffffffffu, send.y, d);
        v[i] = make_float2(keep.x + rx, keep.y + ry);
      }
    }
  }
}

template <typename TS, int T, int MP, bool DZ>
__global__ void __launch_bounds__(PL_THREADS, 1) k_fwd_plane(PlaneArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int S = a.S, NL = a.NL, mL = a.mL, QS = a.QS;
  const PlaneGeom G = plane_geom(S, NL, mL, QS, (int)sizeof(TS), DZ ? 2 : 1);
  constexpr int T2 = 2 * T;                             // threads per row, one pair each
  constexpr int RB = PL_CONSUMERS / T2;
  const int Qs = G.Qs, NS = G.NS, RS = G.RS;
  const int X1S = MP + 1;                               // X1 row stride (float2)
  float2 *X1 = reinterpret_cast<float2 *>(smem + G.x1);
  float2 *twc = reinterpret_cast<float2 *>(smem + G.twc);
  float2 *tw2 = reinterpret_cast<float2 *>(smem + G.tw2);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + G.bar);
  uint64_t *empty = full + PL_MAXSTAGES;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbat = (S + RB - 1) / RB;
  const size_t row_bytes = (size_t)NL * sizeof(TS);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], PL_CONSUMERS / 32);   // every consumer warp frees a stage
    }
    tma::fence_barrier_init();
  }
  // combine table (alpha, beta) per (k, row thread j, pair) and the slab-axis
  // twiddles exp(-2 pi i kq(q) r / S)
  for (int e = tid; e < MP * T * 2; e += PL_THREADS) {
    const int k = e / (2 * T), rem = e - k * 2 * T, j = rem >> 1, pr = rem & 1;
    float2 al = make_float2(0.f, 0.f), be = make_float2(0.f, 0.f);
    if (k < mL) {
      const int ru = 4 * j + 2 * pr, rv = ru + 1;
      double su, cu, sv, cv;
      sincospi(2.0 * (double)((k * ru) % NL) / NL, &su, &cu);
      sincospi(2.0 * (double)((k * rv) % NL) / NL, &sv, &cv);
      al = make_float2((float)(0.5 * (cu - sv)), (float)(-0.5 * (su + cv)));
      be = make_float2((float)(0.5 * (cu + sv)), (float)(0.5 * (cv - su)));
    }
    twc[2 * e] = al;
    twc[2 * e + 1] = be;
  }
  for (int e = tid; e < QS * Qs; e += PL_THREADS) {
    const int q = e / Qs, r = e - q * Qs;
    double sn, cs;
    sincospi(2.0 * (double)mulmod(kept_k(q, a.mS, S), r, S) / S, &sn, &cs);
    tw2[e] = make_float2((float)cs, (float)-sn);
  }
  __syncthreads();

  if (warp == PL_CONSUMERS / 32) {
    // ------------------------------------------------------------ producer
    const TS *in0 = reinterpret_cast<const TS *>(a.in0);
    const TS *in1 = reinterpret_cast<const TS *>(a.in1);
    long long it = 0;
    bool ok = true;
    for (long long plane = blockIdx.x; plane < a.planes && ok; plane += gridDim.x) {
      for (int b = 0; b < nbat; ++b, ++it) {
        const int s = (int)(it % NS);
        if (it >= NS) ok = tc::mbar_wait(&empty[s], (uint32_t)(((it / NS) - 1) & 1), a.err);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        const int rows = min(RB, S - b * RB);
        if (lane == 0)
          tma::arrive_expect_tx(&full[s], (uint32_t)(rows * row_bytes * (DZ ? 2 : 1)));
        __syncwarp();
        unsigned char *st = smem + (size_t)s * G.stage;
        const long long row0 = plane * S + (long long)b * RB;
        // one copy per group of 15 consecutive rows (lane g: group g)
        const int gr = min(PL_WARPS, rows - PL_WARPS * lane);   // rows of group `lane`
        if (lane < G.G && gr > 0) {
          const long long r0 = row0 + (long long)PL_WARPS * lane;
          tma::load_bulk(st + (size_t)lane * G.GS, in0 + r0 * NL, (uint32_t)(gr * row_bytes),
                         &full[s]);
          if (DZ)
            tma::load_bulk(st + (size_t)(G.G + lane) * G.GS, in1 + r0 * NL,
                           (uint32_t)(gr * row_bytes), &full[s]);
        }
        __syncwarp();
      }
    }
    // every issued copy lands before the CTA may exit
    for (long long jt = it - 1; jt >= 0 && jt >= it - NS; --jt)
      tc::mbar_wait(&full[jt % NS], (uint32_t)((jt / NS) & 1), nullptr);
  } else {
    // ------------------------------------------------------------ consumers
    // thread (rl, jj) of a batch owns the subsequences r_u = 4 (jj / 2) + 2 (jj % 2)
    // and r_v = r_u + 1 of row rl: one complex FFT16 of the pair u + i v
    const int grp = (tid & 31) / T2, jj = (tid & 31) - grp * T2;
    const int rl = PL_WARPS * grp + (tid >> 5);          // row of the batch
    const size_t row_off = (size_t)grp * G.GS + (size_t)(tid >> 5) * RS;
    const int Q = NL / 16;
    const float2 *twj = twc + 2 * jj;
    long long it = 0;
    bool ok = true;
    for (long long plane = blockIdx.x; plane < a.planes; plane += gridDim.x) {
      for (int b = 0; b < nbat; ++b, ++it) {
        const int s = (int)(it % NS);
        if (ok) ok = tc::mbar_wait(&full[s], (uint32_t)((it / NS) & 1), a.err);
        ok = __all_sync(0xffffffffu, ok);      // after an expiry: no more waits, same barriers
        const int rows = min(RB, S - b * RB);
        const bool valid = rl < rows;
        const unsigned char *st = smem + (size_t)s * G.stage;
        float2 z[16];
        {
          const TS *src = reinterpret_cast<const TS *>(st + row_off) + 2 * jj;
#pragma unroll
          for (int t = 0; t < 16; ++t) z[t] = valid ? ld_pair(src + t * Q) : make_float2(0.f, 0.f);
          if (DZ) {
            const TS *src1 =
                reinterpret_cast<const TS *>(st + (size_t)G.G * G.GS + row_off) + 2 * jj;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              float2 p = valid ? ld_pair(src1 + t * Q) : make_float2(0.f, 0.f);
              gelu_grad2(p.x, p.y);
              z[t] = make_float2(z[t].x * p.x, z[t].y * p.y);
            }
          } else if (a.tanh_in) {
#pragma unroll
            for (int t = 0; t < 16; ++t) z[t] = make_float2(tanhf(z[t].x), tanhf(z[t].y));
          }
        }
        __syncwarp();
        if (lane == 0) tma::arrive(&empty[s]);       // the stage may be refilled
        fft::fft16<-1>(z);
        float2 acc[MP];
#pragma unroll
        for (int k = 0; k < MP; ++k) acc[k] = make_float2(0.f, 0.f);
        combine_pair<MP>(acc, z, twj, T2);
        rs_lanes<MP, T2>(acc, jj);
        if (valid) {
          float2 *x1r = X1 + (size_t)(b * RB + rl) * X1S + jj * (MP / T2);
#pragma unroll
          for (int i = 0; i < MP / T2; ++i) x1r[i] = acc[i];
        }
      }
      consumers_sync();   // the plane's row spectra are complete
      // slab axis, step 1: FFT16 over a of X1[Qs a + r, k], in place
      for (int task = tid; task < mL * Qs; task += PL_CONSUMERS) {
        const int k = task / Qs, r = task - k * Qs;
        float2 v[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) v[t] = X1[(size_t)(Qs * t + r) * X1S + k];
        fft::fft16<-1>(v);
#pragma unroll
        for (int t = 0; t < 16; ++t) X1[(size_t)(Qs * t + r) * X1S + k] = v[t];
      }
      consumers_sync();
      // step 2: twiddled sums over r for the kept kq only
      float2 *dst = a.out + plane * (long long)(QS * mL);
      for (int task = tid; task < QS * mL; task += PL_CONSUMERS) {
        const int q = task / mL, k = task - q * mL;
        const int p = kept_k(q, a.mS, S) & 15;
        const float2 *zr = X1 + (size_t)(Qs * p) * X1S + k;
        const float2 *tw = tw2 + (size_t)q * Qs;
        float2 sum = make_float2(0.f, 0.f);
        for (int r = 0; r < Qs; ++r) cfma(sum, zr[(size_t)r * X1S], tw[r]);
        dst[task] = sum;
      }
      consumers_sync();   // X1 is free for the next plane
    }
  }
}

template <typename TS, int T, bool DZ>
cudaError_t launch_plane_t(const Launch &L, const PlaneGeom &G, const PlaneArgs &args, int grid) {
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)G.total);
    if (e != cudaSuccess) return e;
    kern<<<grid, PL_THREADS, G.total, L.stream>>>(args);
    return cudaGetLastError();
  };
  switch (G.MP) {
    case 8: return go(k_fwd_plane<TS, T, 8, DZ>);
    case 16: return go(k_fwd_plane<TS, T, 16, DZ>);
    case 24: return go(k_fwd_plane<TS, T, 24, DZ>);
    default: return go(k_fwd_plane<TS, T, 32, DZ>);
  }
}

template <typename TS, bool DZ>
cudaError_t launch_plane_ts(const Launch &L, const PlaneGeom &G, const PlaneArgs &args, int grid) {
  switch (G.T) {
    case 1: return launch_plane_t<TS, 1, DZ>(L, G, args, grid);
    case 2: return launch_plane_t<TS, 2, DZ>(L, G, args, grid);
    case 4: return launch_plane_t<TS, 4, DZ>(L, G, args, grid);
    default: return launch_plane_t<TS, 8, DZ>(L, G, args, grid);
  }
}

}  // namespace

bool fwd_plane_supported(const Geom &g, int dtype, const void *in0, const void *in1,
                         int load_mode) {
  if (g.d < 2 || g.S % 16 != 0) return false;
  if (!(g.NL == 64 || g.NL == 128 || g.NL == 256 || g.NL == 512)) return false;
  if (g.mL > 32 || g.mL > g.NL / 2) return false;
  if ((reinterpret_cast<uintptr_t>(in0) & 15) != 0) return false;
  if (load_mode == LOAD_DZ && (reinterpret_cast<uintptr_t>(in1) & 15) != 0) return false;
  const PlaneGeom G = plane_geom(g.S, g.NL, g.mL, g.QS, dtype == DT_F32 ? 4 : 2,
                                 load_mode == LOAD_DZ ? 2 : 1);
  return G.NS >= 2 && G.total <= PL_SMEM_MAX;
}

cudaError_t launch_fwd_plane(const Launch &L, const Geom &g, int dtype, int load_mode, long long C,
                             const void *in0, const void *in1, float2 *out) {
  const bool dz = load_mode == LOAD_DZ;
  const PlaneGeom G = plane_geom(g.S, g.NL, g.mL, g.QS, dtype == DT_F32 ? 4 : 2, dz ? 2 : 1);
  const long long planes = g.B * C * g.O;
  PlaneArgs args{in0, in1, out, planes, g.S, g.NL, g.mL, g.mS, g.QS,
                 load_mode == LOAD_TANH ? 1 : 0, L.err};
  const int grid = (int)(planes < L.num_sms ? planes : L.num_sms);
  launch_begin(L);
  cudaError_t e;
  if (dtype == DT_F32)
    e = dz ? launch_plane_ts<float, true>(L, G, args, grid)
           : launch_plane_ts<float, false>(L, G, args, grid);
  else if (dtype == DT_F16)
    e = dz ? launch_plane_ts<__half, true>(L, G, args, grid)
           : launch_plane_ts<__half, false>(L, G, args, grid);
  else
    e = dz ? launch_plane_ts<__nv_bfloat16, true>(L, G, args, grid)
           : launch_plane_ts<__nv_bfloat16, false>(L, G, args, grid);
  launch_end(L, dz ? "fwd_plane_dz" : "fwd_plane");
  return e;
}

}  // namespace fno
