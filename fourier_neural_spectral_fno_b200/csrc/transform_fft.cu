// Truncated forward transform (steps S0-S2) as a pruned radix-16 FFT on the
// CUDA cores: the alternative to the dense DFT-matrix contraction of
// transform_pipe.cu / transform_tc.cu, chosen per shape by measurement
// ("Guaranteed approximation bounds and efficient mixed-precision training for
// neural operators", key insights: the block's Fourier transform and
// contraction are memory-bound).
//
// Last axis (length N = 16 Q, keep k < m).  With n = Q a + r,
//     X[k] = sum_r w_N^{k r} Y_r[k mod 16],   Y_r[p] = sum_a x[Q a + r] w_16^{p a},
// w_L = exp(-2 pi i / L): sixteen-point DFTs of the Q stride-Q subsequences
// followed by a twiddled sum that produces only the kept k (a pruned
// decimation-in-time step).  A thread owns four subsequences r = 4j..4j+3 of
// one row (one 16-byte load per a), packs them pairwise into two complex
// sequences u + i v, runs two register FFT16s and folds the real-pair
// separation U = (Z + conj Z')/2, V = (Z - conj Z')/2i into the twiddles:
//     w^{k r_u} U + w^{k r_v} V = Z[m] alpha + conj(Z[-m]) beta,
//     alpha = (w^{k r_u} - i w^{k r_v}) / 2,  beta = (w^{k r_u} + i w^{k r_v}) / 2.
// The T = N/64 threads of a row then reduce-scatter their partial sums with
// warp shuffles, leaving thread j with k in [j MP/T, (j+1) MP/T).
//
// Slab axis: the row spectra of a batch of rows go to shared memory and each
// thread accumulates X2[q, k] = sum_n X1[n, k] exp(-2 pi i kq n / S) for its
// (q, k) pairs directly (the band's rows are few).  A plane's rows are split
// into nb bands, one CTA each, launched as one thread-block cluster; the band
// partials are summed through distributed shared memory and the cluster writes
// the plane's spectrum once (no partial spectra in HBM, no finishing launch).
#include <cooperative_groups.h>

#include "fft16.cuh"
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace cg = cooperative_groups;

namespace fno {

namespace {

constexpr int FT_THREADS = 256;
constexpr int FT_MAXNQ = 4;      // slab-axis modes per thread
constexpr int FT_MAXBANDS = 8;   // portable cluster size

struct FftArgs {
  const void *in0, *in1;   // [planes][S][NL] (in1: pre for LOAD_DZ)
  float2 *out;             // [planes][QS][mL]
  int S, NL, mL, mS, QS;
  int rows_per_band;       // multiple of the batch height
  int load_mode;
};

struct FftPlan {
  int T, RU, MP, KG, QL, NQ, nb, rows_per_band;
  size_t twc, tws, x1, part, total;
};

__host__ __device__ inline size_t al16(size_t v) { return (v + 15) & ~(size_t)15; }
__host__ __device__ inline int mp_of(int mL) { return mL <= 8 ? 8 : mL <= 16 ? 16 : mL <= 24 ? 24 : 32; }

FftPlan fft_plan(const Geom &g) {
  FftPlan p{};
  p.T = g.NL / 64;
  p.RU = FT_THREADS / p.T;
  p.MP = mp_of(g.mL);
  p.KG = p.MP / 2;
  p.QL = FT_THREADS / p.KG;
  p.NQ = (g.QS + p.QL - 1) / p.QL;
  const int batches = (g.S + p.RU - 1) / p.RU;
  int nb = batches < FT_MAXBANDS ? batches : FT_MAXBANDS;
  const int bpb = (batches + nb - 1) / nb;
  p.nb = (batches + bpb - 1) / bpb;
  p.rows_per_band = bpb * p.RU;
  size_t off = 0;
  p.twc = off; off += sizeof(float2) * 4 * (size_t)p.MP * p.T;
  p.tws = off; off += al16(sizeof(float2) * (size_t)g.S);
  p.x1 = off; off += sizeof(float2) * (size_t)p.RU * p.MP;
  p.part = off; off += sizeof(float2) * (size_t)g.QS * p.MP;
  p.total = off;
  return p;
}

template <typename T> struct Vec4;   // four consecutive storage elements
template <> struct Vec4<float> {
  using type = float4;
  static __device__ __forceinline__ float4 unpack(const float4 &v) { return v; }
};
template <> struct Vec4<__half> {
  using type = uint2;
  static __device__ __forceinline__ float4 unpack(const uint2 &v) {
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
};
template <> struct Vec4<__nv_bfloat16> {
  using type = uint2;
  static __device__ __forceinline__ float4 unpack(const uint2 &v) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
};

__device__ __forceinline__ float4 apply_load(float4 v, int mode, float4 p) {
  if (mode == LOAD_TANH) return make_float4(tanhf(v.x), tanhf(v.y), tanhf(v.z), tanhf(v.w));
  if (mode == LOAD_DZ)
    return make_float4(v.x * gelu_grad_f(p.x), v.y * gelu_grad_f(p.y), v.z * gelu_grad_f(p.z),
                       v.w * gelu_grad_f(p.w));
  return v;
}

// Row-spectrum combine table: for mode k, row thread j and pair p, (alpha, beta)
// of the subsequences r_u = 4j + 2p and r_v = r_u + 1 (zero for padded k >= mL).
__device__ void build_combine_table(float2 *twc, int NL, int mL, int MP, int T) {
  for (int e = threadIdx.x; e < MP * T * 2; e += blockDim.x) {
    const int k = e / (2 * T), rem = e - k * 2 * T, j = rem >> 1, p = rem & 1;
    float2 al = make_float2(0.f, 0.f), be = make_float2(0.f, 0.f);
    if (k < mL) {
      const int ru = 4 * j + 2 * p, rv = ru + 1;
      double su, cu, sv, cv;
      sincospi(2.0 * (double)((k * ru) % NL) / NL, &su, &cu);
      sincospi(2.0 * (double)((k * rv) % NL) / NL, &sv, &cv);
      // w^{k r} = c - i s
      al = make_float2((float)(0.5 * (cu - sv)), (float)(-0.5 * (su + cv)));
      be = make_float2((float)(0.5 * (cu + sv)), (float)(0.5 * (cv - su)));
    }
    twc[2 * e] = al;
    twc[2 * e + 1] = be;
  }
}

// acc[k] += Z[m] alpha + conj(Z[-m]) beta, m = k mod 16
template <int MP>
__device__ __forceinline__ void combine(float2 (&acc)[MP], const float2 (&Z)[16],
                                        const float2 *tw, int T) {
#pragma unroll
  for (int k = 0; k < MP; ++k) {
    const int m = k & 15, mm = (16 - m) & 15;
    const float4 ab = *reinterpret_cast<const float4 *>(tw + (size_t)k * T * 4);
    const float2 a = make_float2(ab.x, ab.y), b = make_float2(ab.z, ab.w);
    const float2 z = Z[m], w = Z[mm];
    acc[k].x = fmaf(z.x, a.x, fmaf(-z.y, a.y, fmaf(w.x, b.x, fmaf(w.y, b.y, acc[k].x))));
    acc[k].y = fmaf(z.x, a.y, fmaf(z.y, a.x, fmaf(w.x, b.y, fmaf(-w.y, b.x, acc[k].y))));
  }
}

// Reduce-scatter of MP complex values over T consecutive lanes: afterwards
// lane j of the group holds the sums for k in [j MP/T, (j+1) MP/T) in v[0..).
template <int MP, int T>
__device__ __forceinline__ void reduce_scatter(float2 (&v)[MP], int j) {
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

template <typename TS, int T, int MP>
__global__ void __launch_bounds__(FT_THREADS, (MP <= 16 ? 2 : 1)) k_fwd_fft(FftArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int RU = FT_THREADS / T;
  constexpr int KG = MP / 2;
  constexpr int QL = FT_THREADS / KG;
  const int S = a.S, NL = a.NL, mL = a.mL, QS = a.QS;
  const int Q = NL / 16;
  cg::cluster_group cluster = cg::this_cluster();
  const int nb = (int)cluster.num_blocks();
  const int band = (int)cluster.block_rank();
  const long long plane = blockIdx.x / nb;

  size_t off = 0;
  float2 *twc = reinterpret_cast<float2 *>(smem + off); off += sizeof(float2) * 4 * MP * T;
  float2 *twS = reinterpret_cast<float2 *>(smem + off); off += al16(sizeof(float2) * S);
  float2 *X1 = reinterpret_cast<float2 *>(smem + off); off += sizeof(float2) * RU * MP;
  float2 *part = reinterpret_cast<float2 *>(smem + off);

  build_combine_table(twc, NL, mL, MP, T);
  build_twiddles(twS, S);
  __syncthreads();

  const int tid = threadIdx.x;
  const int rl = tid / T, j = tid - rl * T;          // row in batch, thread of row
  // slab-axis role: k pair kp, q lanes ql + QL s
  const int kp = tid % KG, ql = tid / KG;
  int kq[FT_MAXNQ];
  float2 acc2[FT_MAXNQ][2];
#pragma unroll
  for (int s = 0; s < FT_MAXNQ; ++s) {
    const int q = ql + QL * s;
    kq[s] = q < QS ? (QS == 1 ? 0 : kept_k(q, a.mS, S)) : 0;
    acc2[s][0] = acc2[s][1] = make_float2(0.f, 0.f);
  }

  using V = Vec4<TS>;
  using VT = typename V::type;
  const TS *in0 = reinterpret_cast<const TS *>(a.in0) + plane * (long long)S * NL;
  const TS *in1 = a.load_mode == LOAD_DZ
                      ? reinterpret_cast<const TS *>(a.in1) + plane * (long long)S * NL
                      : nullptr;
  const int r_begin = band * a.rows_per_band;
  const int r_end = min(S, r_begin + a.rows_per_band);
  const float2 *twj = twc + j * 4;

  for (int r0 = r_begin; r0 < r_end; r0 += RU) {
    const int row = r0 + rl;
    const bool valid = row < r_end;
    float2 acc[MP];
#pragma unroll
    for (int k = 0; k < MP; ++k) acc[k] = make_float2(0.f, 0.f);
    {
      float4 xv[16];
      const VT *src = reinterpret_cast<const VT *>(in0 + (long long)row * NL + 4 * j);
      const VT *src1 = in1 ? reinterpret_cast<const VT *>(in1 + (long long)row * NL + 4 * j)
                           : nullptr;
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        VT raw{};
        if (valid) raw = __ldg(src + (size_t)t * (Q / 4));
        xv[t] = V::unpack(raw);
      }
      if (a.load_mode != LOAD_PLAIN) {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          float4 pv = make_float4(0.f, 0.f, 0.f, 0.f);
          if (a.load_mode == LOAD_DZ && valid) pv = V::unpack(__ldg(src1 + (size_t)t * (Q / 4)));
          xv[t] = apply_load(xv[t], a.load_mode, pv);
        }
      }
      float2 z[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) z[t] = make_float2(xv[t].x, xv[t].y);
      fft::fft16<-1>(z);
      combine<MP>(acc, z, twj, T);
#pragma unroll
      for (int t = 0; t < 16; ++t) z[t] = make_float2(xv[t].z, xv[t].w);
      fft::fft16<-1>(z);
      combine<MP>(acc, z, twj + 2, T);
    }
    reduce_scatter<MP, T>(acc, j);
    __syncthreads();   // the previous batch's slab-axis pass is done with X1
#pragma unroll
    for (int i = 0; i < MP / T; ++i) X1[rl * MP + j * (MP / T) + i] = acc[i];
    __syncthreads();
    const int nrows = min(RU, r_end - r0);
#pragma unroll
    for (int s = 0; s < FT_MAXNQ; ++s) {
      if (s < (QS + QL - 1) / QL && ql + QL * s < QS) {
        int idx = mulmod(kq[s], r0, S);
        float2 s0 = acc2[s][0], s1 = acc2[s][1];
        for (int n = 0; n < nrows; ++n) {
          const float4 xx = *reinterpret_cast<const float4 *>(X1 + n * MP + 2 * kp);
          const float2 w = twS[idx];
          cfma_conj_b(s0, make_float2(xx.x, xx.y), w);
          cfma_conj_b(s1, make_float2(xx.z, xx.w), w);
          idx += kq[s];
          if (idx >= S) idx -= S;
        }
        acc2[s][0] = s0;
        acc2[s][1] = s1;
      }
    }
  }
  // band partial -> shared memory, then the cluster sums the bands
#pragma unroll
  for (int s = 0; s < FT_MAXNQ; ++s) {
    const int q = ql + QL * s;
    if (q < QS) {
      part[q * MP + 2 * kp] = acc2[s][0];
      part[q * MP + 2 * kp + 1] = acc2[s][1];
    }
  }
  cluster.sync();
  const int P = QS * mL;
  float2 *dst = a.out + plane * (long long)P;
  for (int p = band * FT_THREADS + tid; p < P; p += nb * FT_THREADS) {
    const int q = p / mL, k = p - q * mL;
    float2 sum = make_float2(0.f, 0.f);
    for (int r = 0; r < nb; ++r) {
      const float2 *rp = cluster.map_shared_rank(part, r);
      const float2 v = rp[q * MP + k];
      sum.x += v.x;
      sum.y += v.y;
    }
    dst[p] = sum;
  }
  cluster.sync();   // no CTA leaves while another reads its shared memory
}

template <typename TS, int T>
cudaError_t launch_fft_t(const Launch &L, const FftPlan &p, const FftArgs &args,
                         long long planes) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(planes * p.nb));
  cfg.blockDim = dim3(FT_THREADS);
  cfg.dynamicSmemBytes = p.total;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.nb;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)p.total);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, kern, args);
  };
  switch (p.MP) {
    case 8: return go(k_fwd_fft<TS, T, 8>);
    case 16: return go(k_fwd_fft<TS, T, 16>);
    case 24: return go(k_fwd_fft<TS, T, 24>);
    default: return go(k_fwd_fft<TS, T, 32>);
  }
}

template <typename TS>
cudaError_t launch_fft_ts(const Launch &L, const FftPlan &p, const FftArgs &args,
                          long long planes) {
  switch (p.T) {
    case 1: return launch_fft_t<TS, 1>(L, p, args, planes);
    case 2: return launch_fft_t<TS, 2>(L, p, args, planes);
    case 4: return launch_fft_t<TS, 4>(L, p, args, planes);
    default: return launch_fft_t<TS, 8>(L, p, args, planes);
  }
}

}  // namespace

bool fwd_fft_supported(const Geom &g, const void *in0, const void *in1, int load_mode) {
  if (g.d < 2) return false;                                  // 1D: one row per plane
  if (!(g.NL == 64 || g.NL == 128 || g.NL == 256 || g.NL == 512)) return false;
  if (g.mL > 32 || g.mL > g.NL / 2) return false;
  if ((reinterpret_cast<uintptr_t>(in0) & 15) != 0) return false;
  if (load_mode == LOAD_DZ && (reinterpret_cast<uintptr_t>(in1) & 15) != 0) return false;
  const FftPlan p = fft_plan(g);
  if (p.NQ > FT_MAXNQ) return false;
  if (g.B * g.O > (1LL << 24)) return false;
  return p.total <= 200 * 1024;
}

cudaError_t launch_fwd_fft(const Launch &L, const Geom &g, int dtype, int load_mode, long long C,
                           const void *in0, const void *in1, float2 *out) {
  const FftPlan p = fft_plan(g);
  const long long planes = g.B * C * g.O;
  FftArgs args{in0, in1, out, g.S, g.NL, g.mL, g.mS, g.QS, p.rows_per_band, load_mode};
  launch_begin(L);
  cudaError_t e;
  if (dtype == DT_F32) e = launch_fft_ts<float>(L, p, args, planes);
  else if (dtype == DT_F16) e = launch_fft_ts<__half>(L, p, args, planes);
  else e = launch_fft_ts<__nv_bfloat16>(L, p, args, planes);
  launch_end(L, load_mode == LOAD_DZ ? "fwd_fft_dz" : "fwd_fft");
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fno
