// Pointwise network stages around the spectral blocks (step S5): the lifting
// v = P a + p, the projection u = Q2 GELU(Q1 v + q1) + q2, their adjoints,
// and the mean-squared-error loss of the training step.
//
// One thread owns one grid point.  Parameter gradients are reduced per CTA in
// shared memory over a persistent loop of point tiles and written as per-CTA
// partials, which a second kernel sums in a fixed order (deterministic).
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int NT = 256;      // threads of the forward pointwise kernels
constexpr int PB = 128;      // points per tile of the backward kernels
constexpr int HC = 32;       // projection hidden units per chunk
constexpr int kMaxIn = 8;    // lift input channels
constexpr int kMaxOut = 4;   // projection output channels

template <typename T>
__global__ void __launch_bounds__(NT)
    k_lift(const T *__restrict__ a, const T *__restrict__ P, const T *__restrict__ p,
           T *__restrict__ v, long long B, long long N, int in_ch, int width) {
  __shared__ float Ps[kMaxWidth * kMaxIn], ps[kMaxWidth];
  for (int e = threadIdx.x; e < width * in_ch; e += NT) Ps[e] = to_f<T>(P[e]);
  for (int e = threadIdx.x; e < width; e += NT) ps[e] = to_f<T>(p[e]);
  __syncthreads();
  for (long long t = (long long)blockIdx.x * NT + threadIdx.x; t < B * N;
       t += (long long)gridDim.x * NT) {
    const long long b = t / N, n = t - b * N;
    float aj[kMaxIn];
#pragma unroll
    for (int j = 0; j < kMaxIn; ++j) aj[j] = j < in_ch ? ldf<T>(a + (b * in_ch + j) * N + n) : 0.f;
    for (int c = 0; c < width; ++c) {
      float s = ps[c];
#pragma unroll
      for (int j = 0; j < kMaxIn; ++j)
        if (j < in_ch) s = fmaf(Ps[c * in_ch + j], aj[j], s);
      v[(b * width + c) * N + n] = from_f<T>(s);
    }
  }
}

// Lift for rows whose length is a multiple of 4: a thread takes 4 consecutive
// points, loads each input channel as one vector, and writes each of the width
// output channels as one vector (weights broadcast from shared memory).
template <typename T> struct Vec4;
template <> struct Vec4<float> {
  using raw = float4;
  __device__ static void load(const float *p, float (&v)[4]) {
    const float4 r = *reinterpret_cast<const float4 *>(p);
    v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w;
  }
  __device__ static void store(float *p, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <typename T> struct Vec4 {   // 16-bit storage: 8-byte vectors
  __device__ static void load(const T *p, float (&v)[4]) {
    const uint2 r = *reinterpret_cast<const uint2 *>(p);
    const T *h = reinterpret_cast<const T *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = to_f<T>(h[i]);
  }
  __device__ static void store(T *p, const float (&v)[4]) {
    uint2 r;
    T *h = reinterpret_cast<T *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = from_f<T>(v[i]);
    *reinterpret_cast<uint2 *>(p) = r;
  }
};

template <typename T>
__global__ void __launch_bounds__(NT)
    k_lift4(const T *__restrict__ a, const T *__restrict__ P, const T *__restrict__ p,
            T *__restrict__ v, long long B, long long N, int in_ch, int width) {
  __shared__ float Ps[kMaxWidth * kMaxIn], ps[kMaxWidth];
  for (int e = threadIdx.x; e < width * in_ch; e += NT) Ps[e] = to_f<T>(P[e]);
  for (int e = threadIdx.x; e < width; e += NT) ps[e] = to_f<T>(p[e]);
  __syncthreads();
  const long long N4 = N / 4;
  for (long long t = (long long)blockIdx.x * NT + threadIdx.x; t < B * N4;
       t += (long long)gridDim.x * NT) {
    const long long b = t / N4, n = (t - b * N4) * 4;
    float x[kMaxIn][4];
    const T *ap = a + b * in_ch * N + n;
#pragma unroll
    for (int j = 0; j < kMaxIn; ++j) {
      if (j < in_ch) Vec4<T>::load(ap + j * N, x[j]);
    }
    T *vp = v + b * width * N + n;
    const float *pw = Ps;
    for (int c = 0; c < width; ++c) {
      float o[4];
      const float bc = ps[c];
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = bc;
#pragma unroll
      for (int j = 0; j < kMaxIn; ++j) {
        if (j < in_ch) {
          const float w = pw[j];
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] = fmaf(w, x[j][i], o[i]);
        }
      }
      pw += in_ch;
      Vec4<T>::store(vp, o);
      vp += N;
    }
  }
}

template <typename T, int CMAX>
__global__ void __launch_bounds__(NT)
    k_proj_fwd(const T *__restrict__ v, const T *__restrict__ Q1, const T *__restrict__ q1,
               const T *__restrict__ Q2, const T *__restrict__ q2, T *__restrict__ u, long long B,
               long long N, int width, int hidden, int out_ch) {
  extern __shared__ __align__(16) float psm[];
  const int ld = (width + 3) & ~3;
  float *Q1s = psm;                    // [hidden][ld]
  float *q1s = Q1s + hidden * ld;      // [hidden]
  float *Q2s = q1s + hidden;           // [out][hidden]
  for (int e = threadIdx.x; e < hidden * ld; e += NT) {
    const int h = e / ld, c = e - h * ld;
    Q1s[e] = c < width ? to_f<T>(Q1[h * width + c]) : 0.f;
  }
  for (int e = threadIdx.x; e < hidden; e += NT) q1s[e] = to_f<T>(q1[e]);
  for (int e = threadIdx.x; e < out_ch * hidden; e += NT) Q2s[e] = to_f<T>(Q2[e]);
  __syncthreads();
  for (long long t = (long long)blockIdx.x * NT + threadIdx.x; t < B * N;
       t += (long long)gridDim.x * NT) {
    const long long b = t / N, n = t - b * N;
    float vr[CMAX];
#pragma unroll
    for (int c = 0; c < CMAX; ++c) vr[c] = c < width ? ldf<T>(v + (b * width + c) * N + n) : 0.f;
    float uo[kMaxOut];
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o) uo[o] = o < out_ch ? to_f<T>(q2[o]) : 0.f;
    for (int h = 0; h < hidden; ++h) {
      const float4 *qp = reinterpret_cast<const float4 *>(Q1s + h * ld);
      float z = q1s[h];
#pragma unroll
      for (int c4 = 0; c4 < CMAX / 4; ++c4) {
        if (4 * c4 < width) {
          const float4 q = qp[c4];
          z = fmaf(q.x, vr[4 * c4], z);
          z = fmaf(q.y, vr[4 * c4 + 1], z);
          z = fmaf(q.z, vr[4 * c4 + 2], z);
          z = fmaf(q.w, vr[4 * c4 + 3], z);
        }
      }
      const float gz = gelu_f(z);
#pragma unroll
      for (int o = 0; o < kMaxOut; ++o)
        if (o < out_ch) uo[o] = fmaf(Q2s[o * hidden + h], gz, uo[o]);
    }
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o)
      if (o < out_ch) u[(b * out_ch + o) * N + n] = from_f<T>(uo[o]);
  }
}

struct ProjBwdLayout {
  size_t Q1s, q1s, Q2s, vs, dus, dhs, gs, acc1, acc2, total;
  int ld;
};

__host__ __device__ inline ProjBwdLayout proj_bwd_layout(int width, int hidden, int out_ch) {
  ProjBwdLayout l;
  l.ld = (width + 3) & ~3;
  size_t off = 0;
  l.Q1s = off; off += sizeof(float) * (size_t)hidden * l.ld;
  l.q1s = off; off += sizeof(float) * hidden;
  l.Q2s = off; off += sizeof(float) * (size_t)out_ch * hidden;
  // v rows: width channels, the ones row, and pad rows up to a multiple of 4
  // (read only by dQ1 blocks whose entries are discarded)
  const int vrows = ((width + 3) & ~3) > width + 1 ? ((width + 3) & ~3) : width + 1;
  l.vs = off; off += sizeof(float) * (size_t)vrows * (PB + 1);
  l.dus = off; off += sizeof(float) * (size_t)out_ch * PB;
  l.dhs = off; off += sizeof(float) * (size_t)HC * PB;
  l.gs = off; off += sizeof(float) * (size_t)HC * (PB + 1);
  l.acc1 = off; off += sizeof(float) * (size_t)hidden * (width + 1);
  l.acc2 = off; off += sizeof(float) * (size_t)out_ch * (hidden + 1);
  l.total = (off + 15) & ~(size_t)15;
  return l;
}

// Projection adjoint: dv, and per-CTA partials of dQ1|dq1 ([hidden][width+1])
// followed by dQ2|dq2 ([out][hidden+1]).  Two threads per point of a tile,
// each taking half of every hidden chunk; their dv contributions meet in
// shared memory at the end of the tile.
constexpr int PBT = 2 * PB;   // threads of k_proj_bwd
template <typename T, int CMAX>
__global__ void __launch_bounds__(PBT)
    k_proj_bwd(const T *__restrict__ v, const T *__restrict__ du, const T *__restrict__ Q1,
               const T *__restrict__ q1, const T *__restrict__ Q2, T *__restrict__ dv,
               float *__restrict__ partial, long long B, long long N, int width, int hidden,
               int out_ch) {
  extern __shared__ __align__(16) unsigned char smem[];
  const ProjBwdLayout lay = proj_bwd_layout(width, hidden, out_ch);
  const int ld = lay.ld;
  float *Q1s = reinterpret_cast<float *>(smem + lay.Q1s);
  float *q1s = reinterpret_cast<float *>(smem + lay.q1s);
  float *Q2s = reinterpret_cast<float *>(smem + lay.Q2s);
  float *v_s = reinterpret_cast<float *>(smem + lay.vs);
  float *du_s = reinterpret_cast<float *>(smem + lay.dus);
  float *dh_s = reinterpret_cast<float *>(smem + lay.dhs);
  float *g_s = reinterpret_cast<float *>(smem + lay.gs);
  float *acc1 = reinterpret_cast<float *>(smem + lay.acc1);
  float *acc2 = reinterpret_cast<float *>(smem + lay.acc2);
  const int tid = threadIdx.x;
  const int pt = tid & (PB - 1), half = tid / PB;   // point of the tile, hidden half
  for (int e = tid; e < hidden * ld; e += PBT) {
    const int h = e / ld, c = e - h * ld;
    Q1s[e] = c < width ? to_f<T>(Q1[h * width + c]) : 0.f;
  }
  for (int e = tid; e < hidden; e += PBT) q1s[e] = to_f<T>(q1[e]);
  for (int e = tid; e < out_ch * hidden; e += PBT) Q2s[e] = to_f<T>(Q2[e]);
  for (int e = tid; e < hidden * (width + 1); e += PBT) acc1[e] = 0.f;
  for (int e = tid; e < out_ch * (hidden + 1); e += PBT) acc2[e] = 0.f;

  const long long total = B * N;
  const long long ntiles = (total + PB - 1) / PB;
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const long long t = tile * PB + pt;
    const bool valid = t < total;
    const long long b = valid ? t / N : 0, n = valid ? t - b * N : 0;
    __syncthreads();
    float vr[CMAX], dvr[CMAX];
#pragma unroll
    for (int c = 0; c < CMAX; ++c) {
      vr[c] = (valid && c < width) ? ldf<T>(v + (b * width + c) * N + n) : 0.f;
      dvr[c] = 0.f;
      if (c < width && half == 0) v_s[c * (PB + 1) + pt] = vr[c];
    }
    if (half == 0) v_s[width * (PB + 1) + pt] = valid ? 1.f : 0.f;
    float dur[kMaxOut];
#pragma unroll
    for (int o = 0; o < kMaxOut; ++o) {
      dur[o] = (valid && o < out_ch) ? ldf<T>(du + (b * out_ch + o) * N + n) : 0.f;
      if (o < out_ch && half == 0) du_s[o * PB + pt] = dur[o];
    }
    for (int hc = 0; hc < hidden; hc += HC) {
      __syncthreads();  // previous chunk's reductions are done with dh_s / g_s
      for (int hh = half * (HC / 2); hh < (half + 1) * (HC / 2); ++hh) {
        const int h = hc + hh;
        float dh = 0.f, gz = 0.f;
        if (h < hidden && valid) {
          const float4 *qp = reinterpret_cast<const float4 *>(Q1s + h * ld);
          // four independent partial sums keep the FMA pipe busy
          float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
          for (int c4 = 0; c4 < CMAX / 4; ++c4) {
            if (4 * c4 < width) {
              const float4 q = qp[c4];
              z0 = fmaf(q.x, vr[4 * c4], z0);
              z1 = fmaf(q.y, vr[4 * c4 + 1], z1);
              z2 = fmaf(q.z, vr[4 * c4 + 2], z2);
              z3 = fmaf(q.w, vr[4 * c4 + 3], z3);
            }
          }
          const float z = q1s[h] + ((z0 + z1) + (z2 + z3));
          float gp;
          gelu_and_grad_f(z, gz, gp);
          float dg = 0.f;
#pragma unroll
          for (int o = 0; o < kMaxOut; ++o)
            if (o < out_ch) dg = fmaf(Q2s[o * hidden + h], dur[o], dg);
          dh = dg * gp;
#pragma unroll
          for (int c4 = 0; c4 < CMAX / 4; ++c4) {
            if (4 * c4 < width) {
              const float4 q = qp[c4];
              dvr[4 * c4] = fmaf(q.x, dh, dvr[4 * c4]);
              dvr[4 * c4 + 1] = fmaf(q.y, dh, dvr[4 * c4 + 1]);
              dvr[4 * c4 + 2] = fmaf(q.z, dh, dvr[4 * c4 + 2]);
              dvr[4 * c4 + 3] = fmaf(q.w, dh, dvr[4 * c4 + 3]);
            }
          }
        }
        dh_s[hh * PB + pt] = dh;
        g_s[hh * (PB + 1) + pt] = gz;
      }
      __syncthreads();
      const int hn = min(HC, hidden - hc);
      {
        // dQ1[h][c] over this tile's points as 4 x 4 blocks (h, c) per thread:
        // 8 shared-memory loads feed 16 multiply-adds per point
        constexpr int HB = 4, CB = 4;
        const int ncb = (width + CB - 1) / CB;
        const int nblk = ((hn + HB - 1) / HB) * ncb;
        // (dh rows past the chunk are zeros; v pad rows only reach discarded
        // entries, so the loads need no guards)
        for (int blk = tid; blk < nblk; blk += PBT) {
          const int hb = blk / ncb, cb = blk - hb * ncb;
          const float *dp = dh_s + hb * HB * PB;
          const float *vp = v_s + cb * CB * (PB + 1);
          float acc[HB][CB];
#pragma unroll
          for (int i = 0; i < HB; ++i)
#pragma unroll
            for (int j = 0; j < CB; ++j) acc[i][j] = 0.f;
#pragma unroll 4
          for (int k = 0; k < PB; ++k) {
            float dv4[HB], v4[CB];
#pragma unroll
            for (int i = 0; i < HB; ++i) dv4[i] = dp[i * PB + k];
#pragma unroll
            for (int j = 0; j < CB; ++j) v4[j] = vp[j * (PB + 1) + k];
#pragma unroll
            for (int i = 0; i < HB; ++i)
#pragma unroll
              for (int j = 0; j < CB; ++j) acc[i][j] = fmaf(dv4[i], v4[j], acc[i][j]);
          }
#pragma unroll
          for (int i = 0; i < HB; ++i)
#pragma unroll
            for (int j = 0; j < CB; ++j)
              if (hb * HB + i < hn && cb * CB + j < width)
                acc1[(hc + hb * HB + i) * (width + 1) + cb * CB + j] += acc[i][j];
        }
        // bias column dq1[h] = sum_p dh[h][p] and dQ2[o][h] = sum_p du[o][p]
        // g[h][p], on the highest threads (idle during the dQ1 blocks), four
        // partial sums each
        for (int e = PBT - 1 - tid; e < hn + out_ch * hn; e += PBT) {
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
          if (e < hn) {
            const float *dr = dh_s + e * PB;
            for (int k = 0; k < PB; k += 4) {
              s0 += dr[k];
              s1 += dr[k + 1];
              s2 += dr[k + 2];
              s3 += dr[k + 3];
            }
            acc1[(hc + e) * (width + 1) + width] += (s0 + s1) + (s2 + s3);
          } else {
            const int o = (e - hn) / hn, hh = e - hn - o * hn;
            const float *dr = du_s + o * PB;
            const float *gr = g_s + hh * (PB + 1);
            for (int k = 0; k < PB; k += 4) {
              s0 = fmaf(dr[k], gr[k], s0);
              s1 = fmaf(dr[k + 1], gr[k + 1], s1);
              s2 = fmaf(dr[k + 2], gr[k + 2], s2);
              s3 = fmaf(dr[k + 3], gr[k + 3], s3);
            }
            acc2[o * (hidden + 1) + hc + hh] += (s0 + s1) + (s2 + s3);
          }
        }
      }
    }
    for (int o = tid; o < out_ch; o += PBT) {
      float s = 0.f;
      for (int k = 0; k < PB; ++k) s += du_s[o * PB + k];
      acc2[o * (hidden + 1) + hidden] += s;
    }
    // the two halves' dv meet in the dh_s / g_s region (free after the last
    // chunk's reductions; it holds CMAX x PB floats)
    __syncthreads();
    float *dvx = dh_s;
    if (half == 1) {
#pragma unroll
      for (int c = 0; c < CMAX; ++c)
        if (c < width) dvx[c * PB + pt] = dvr[c];
    }
    __syncthreads();
    if (half == 0 && valid) {
#pragma unroll
      for (int c = 0; c < CMAX; ++c)
        if (c < width) dv[(b * width + c) * N + n] = from_f<T>(dvr[c] + dvx[c * PB + pt]);
    }
  }
  __syncthreads();
  const long long stride = (long long)hidden * (width + 1) + (long long)out_ch * (hidden + 1);
  float *dst = partial + blockIdx.x * stride;
  for (int e = tid; e < hidden * (width + 1); e += PBT) dst[e] = acc1[e];
  for (int e = tid; e < out_ch * (hidden + 1); e += PBT) dst[hidden * (width + 1) + e] = acc2[e];
}

// Lift adjoint: per-CTA partials of dP|dp ([width][in+1]).
template <typename T>
__global__ void __launch_bounds__(PB)
    k_lift_bwd(const T *__restrict__ a, const T *__restrict__ dv, float *__restrict__ partial,
               long long B, long long N, int in_ch, int width) {
  __shared__ float dv_s[kMaxWidth * PB];
  __shared__ float a_s[(kMaxIn + 1) * (PB + 1)];
  __shared__ float acc[kMaxWidth * (kMaxIn + 1)];
  const int tid = threadIdx.x;
  for (int e = tid; e < width * (in_ch + 1); e += PB) acc[e] = 0.f;
  const long long total = B * N;
  const long long ntiles = (total + PB - 1) / PB;
  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const long long t = tile * PB + tid;
    const bool valid = t < total;
    const long long b = valid ? t / N : 0, n = valid ? t - b * N : 0;
    __syncthreads();
    for (int c = 0; c < width; ++c)
      dv_s[c * PB + tid] = valid ? ldf<T>(dv + (b * width + c) * N + n) : 0.f;
    for (int j = 0; j < in_ch; ++j)
      a_s[j * (PB + 1) + tid] = valid ? ldf<T>(a + (b * in_ch + j) * N + n) : 0.f;
    a_s[in_ch * (PB + 1) + tid] = valid ? 1.f : 0.f;
    __syncthreads();
    for (int e = tid; e < width * (in_ch + 1); e += PB) {
      const int c = e / (in_ch + 1), j = e - c * (in_ch + 1);
      float s = 0.f;
      for (int k = 0; k < PB; ++k) s = fmaf(dv_s[c * PB + k], a_s[j * (PB + 1) + k], s);
      acc[e] += s;
    }
  }
  __syncthreads();
  for (int e = tid; e < width * (in_ch + 1); e += PB)
    partial[(long long)blockIdx.x * width * (in_ch + 1) + e] = acc[e];
}

// Lift adjoint, streaming form (the same per-CTA partials): warp w owns the
// eight channels of group w % NCG and keeps their [8][IN + 1] sums in
// registers; its lanes walk chunks of 16 bytes of consecutive points (8 for
// 16-bit storage, 4 for float32) of one sample, all eight channel loads and the
// IN input loads of a chunk in flight at once.  Lanes, then the warps of a
// point group, meet once at the end (shuffles, then shared memory), in a fixed
// order.  The tiled kernel above waited out one load per channel per tile.
constexpr int LB_THREADS = 256, LB_CPW = 8;

template <typename T> struct Pack16 {   // 16 bytes of storage elements
  static constexpr int n = 16 / (int)sizeof(T);
};
template <typename T>
__device__ __forceinline__ void unpack16(const uint4 &r, float (&v)[Pack16<T>::n]) {
  if constexpr (sizeof(T) == 4) {
    v[0] = __uint_as_float(r.x);
    v[1] = __uint_as_float(r.y);
    v[2] = __uint_as_float(r.z);
    v[3] = __uint_as_float(r.w);
  } else {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const T lo = *reinterpret_cast<const T *>(reinterpret_cast<const unsigned short *>(&w[i]));
      const T hi =
          *reinterpret_cast<const T *>(reinterpret_cast<const unsigned short *>(&w[i]) + 1);
      v[2 * i] = to_f<T>(lo);
      v[2 * i + 1] = to_f<T>(hi);
    }
  }
}

template <typename T, int IN>
__global__ void __launch_bounds__(LB_THREADS)
    k_lift_bwd16(const T *__restrict__ a, const T *__restrict__ dv, float *__restrict__ partial,
                 long long B, long long N, int width, int ncg) {
  constexpr int PP = Pack16<T>::n;            // points per chunk
  constexpr int NW = LB_THREADS / 32;
  __shared__ float red[NW][LB_CPW * (IN + 1)];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int npg = NW / ncg, cg = warp % ncg, pg = warp / ncg;
  const int c0 = cg * LB_CPW;
  float acc[LB_CPW][IN + 1];
#pragma unroll
  for (int c = 0; c < LB_CPW; ++c)
#pragma unroll
    for (int j = 0; j <= IN; ++j) acc[c][j] = 0.f;
  const long long nchunk = B * N / PP;
  if (pg < npg) {
    const long long step = (long long)gridDim.x * npg * 32;
    for (long long q = ((long long)blockIdx.x * npg + pg) * 32 + lane; q < nchunk; q += step) {
      const long long t = q * PP, b = t / N, n = t - b * N;
      uint4 ar[IN], dr[LB_CPW];
#pragma unroll
      for (int j = 0; j < IN; ++j)
        ar[j] = __ldg(reinterpret_cast<const uint4 *>(a + (b * IN + j) * N + n));
#pragma unroll
      for (int c = 0; c < LB_CPW; ++c)
        dr[c] = c0 + c < width
                    ? __ldg(reinterpret_cast<const uint4 *>(dv + (b * width + c0 + c) * N + n))
                    : make_uint4(0u, 0u, 0u, 0u);
      float av[IN][PP];
#pragma unroll
      for (int j = 0; j < IN; ++j) unpack16<T>(ar[j], av[j]);
#pragma unroll
      for (int c = 0; c < LB_CPW; ++c) {
        float d[PP];
        unpack16<T>(dr[c], d);
#pragma unroll
        for (int i = 0; i < PP; ++i) {
#pragma unroll
          for (int j = 0; j < IN; ++j) acc[c][j] = fmaf(d[i], av[j][i], acc[c][j]);
          acc[c][IN] += d[i];
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < LB_CPW; ++c)
#pragma unroll
    for (int j = 0; j <= IN; ++j) {
      float v = acc[c][j];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) red[warp][c * (IN + 1) + j] = v;
    }
  __syncthreads();
  for (int e = threadIdx.x; e < width * (IN + 1); e += LB_THREADS) {
    const int c = e / (IN + 1), j = e - c * (IN + 1);
    const int g = c / LB_CPW, cc = c - g * LB_CPW;
    float v = 0.f;
    for (int p2 = 0; p2 < npg; ++p2) v += red[p2 * ncg + g][cc * (IN + 1) + j];
    partial[(long long)blockIdx.x * width * (IN + 1) + e] = v;
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
    k_mse(const T *__restrict__ u, const T *__restrict__ tg, float *__restrict__ loss,
          T *__restrict__ du, long long n) {
  __shared__ float red[8];
  const float inv_n = 1.0f / (float)n;
  float s = 0.f;
  for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < n;
       i += (long long)gridDim.x * 256) {
    const float d = ldf<T>(u + i) - ldf<T>(tg + i);
    s = fmaf(d, d, s);
    if (du) du[i] = from_f<T>(2.0f * d * inv_n);
  }
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    atomicAdd(loss, t * inv_n);
  }
}

int pointwise_grid(long long total, int num_sms) {
  const long long want = (total + NT - 1) / NT;
  const long long cap = (long long)num_sms * 16;
  return (int)(want < cap ? want : cap);
}

}  // namespace

#define FNO_DISPATCH_T(dtype, ...)                                \
  do {                                                            \
    if ((dtype) == DT_F32) {                                      \
      using T = float;                                            \
      __VA_ARGS__;                                                \
    } else if ((dtype) == DT_F16) {                               \
      using T = __half;                                           \
      __VA_ARGS__;                                                \
    } else {                                                      \
      using T = __nv_bfloat16;                                    \
      __VA_ARGS__;                                                \
    }                                                             \
  } while (0)

cudaError_t launch_lift(const Launch &L, const Geom &g, int dtype, int in_ch, int width,
                        const void *a, const void *P, const void *p, void *v) {
  const size_t vb = dtype == DT_F32 ? 16 : 8;   // vector bytes of 4 elements
  const bool vec = g.N % 4 == 0 && (reinterpret_cast<uintptr_t>(a) % vb) == 0 &&
                   (reinterpret_cast<uintptr_t>(v) % vb) == 0;
  launch_begin(L);
  if (vec) {
    const int grid = pointwise_grid(g.B * g.N / 4, L.num_sms);
    FNO_DISPATCH_T(dtype, k_lift4<T><<<grid, NT, 0, L.stream>>>(
                              (const T *)a, (const T *)P, (const T *)p, (T *)v, g.B, g.N, in_ch,
                              width));
  } else {
    const int grid = pointwise_grid(g.B * g.N, L.num_sms);
    FNO_DISPATCH_T(dtype, k_lift<T><<<grid, NT, 0, L.stream>>>(
                              (const T *)a, (const T *)P, (const T *)p, (T *)v, g.B, g.N, in_ch,
                              width));
  }
  launch_end(L, "lift");
  return cudaGetLastError();
}

template <typename T, int CMAX>
static cudaError_t proj_fwd_t(const Launch &L, const Geom &g, int width, int hidden, int out_ch,
                              const void *v, const void *Q1, const void *q1, const void *Q2,
                              const void *q2, void *u) {
  const int ld = (width + 3) & ~3;
  const size_t smem = sizeof(float) * ((size_t)hidden * ld + hidden + (size_t)out_ch * hidden);
  auto kern = k_proj_fwd<T, CMAX>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  kern<<<pointwise_grid(g.B * g.N, L.num_sms), NT, smem, L.stream>>>(
      (const T *)v, (const T *)Q1, (const T *)q1, (const T *)Q2, (const T *)q2, (T *)u, g.B, g.N,
      width, hidden, out_ch);
  return cudaGetLastError();
}

cudaError_t launch_proj_fwd(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                            int out_ch, const void *v, const void *Q1, const void *q1,
                            const void *Q2, const void *q2, void *u) {
  if ((L.tc == 1 || L.tc == 3 || L.tc == 4) && proj_pipe_supported(g, dtype, width, hidden, out_ch, v))
    return launch_proj_pipe(L, g, dtype, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
  if (L.tc && proj_tc_supported(g, dtype, width, hidden, out_ch))
    return launch_proj_fwd_tc(L, g, dtype, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
  cudaError_t err;
  launch_begin(L);
  FNO_DISPATCH_T(dtype, {
    if (width <= 16)
      err = proj_fwd_t<T, 16>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
    else if (width <= 32)
      err = proj_fwd_t<T, 32>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
    else
      err = proj_fwd_t<T, 64>(L, g, width, hidden, out_ch, v, Q1, q1, Q2, q2, u);
  });
  launch_end(L, "proj_fwd");
  return err;
}

int proj_bwd_grid(const Geom &g, int num_sms) {
  const long long ntiles = (g.B * g.N + PB - 1) / PB;
  const long long cap = kPartialCTAs;
  return (int)(ntiles < cap ? ntiles : cap);
}

size_t proj_bwd_partial_floats(int width, int hidden, int out_ch) {
  return (size_t)hidden * (width + 1) + (size_t)out_ch * (hidden + 1);
}

size_t proj_bwd_smem_bytes(int width, int hidden, int out_ch) {
  return proj_bwd_layout(width, hidden, out_ch).total;
}

template <typename T, int CMAX>
static cudaError_t proj_bwd_t(const Launch &L, const Geom &g, int width, int hidden, int out_ch,
                              const void *v, const void *du, const void *Q1, const void *q1,
                              const void *Q2, void *dv, float *partial, int grid) {
  const size_t smem = proj_bwd_layout(width, hidden, out_ch).total;
  auto kern = k_proj_bwd<T, CMAX>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  kern<<<grid, PBT, smem, L.stream>>>((const T *)v, (const T *)du, (const T *)Q1, (const T *)q1,
                                     (const T *)Q2, (T *)dv, partial, g.B, g.N, width, hidden,
                                     out_ch);
  return cudaGetLastError();
}

cudaError_t launch_proj_bwd(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                            int out_ch, const void *v, const void *du, const void *Q1,
                            const void *q1, const void *Q2, void *dv, float *partial) {
  const int grid = proj_bwd_grid(g, L.num_sms);
  cudaError_t err;
  launch_begin(L);
  FNO_DISPATCH_T(dtype, {
    if (width <= 16)
      err = proj_bwd_t<T, 16>(L, g, width, hidden, out_ch, v, du, Q1, q1, Q2, dv, partial, grid);
    else if (width <= 32)
      err = proj_bwd_t<T, 32>(L, g, width, hidden, out_ch, v, du, Q1, q1, Q2, dv, partial, grid);
    else
      err = proj_bwd_t<T, 64>(L, g, width, hidden, out_ch, v, du, Q1, q1, Q2, dv, partial, grid);
  });
  launch_end(L, "proj_bwd");
  return err;
}

int lift_bwd_grid(const Geom &g, int num_sms) {
  const long long ntiles = (g.B * g.N + PB - 1) / PB;
  const long long cap = kPartialCTAs;
  return (int)(ntiles < cap ? ntiles : cap);
}

cudaError_t launch_lift_bwd(const Launch &L, const Geom &g, int dtype, int in_ch, int width,
                            const void *a, const void *dv, float *partial) {
  const int grid = lift_bwd_grid(g, L.num_sms);
  // the streaming form: 16-byte chunks of points that stay inside a sample,
  // 16-byte aligned rows, at most 64 channels, 2 to 4 inputs
  const int pp = dtype == DT_F32 ? 4 : 8;
  const bool stream16 = g.N % pp == 0 && width <= 64 && in_ch >= 2 && in_ch <= 4 &&
                        ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(dv)) & 15) == 0;
  const int groups = (width + LB_CPW - 1) / LB_CPW;
  const int ncg = groups <= 1 ? 1 : groups <= 2 ? 2 : groups <= 4 ? 4 : 8;
  launch_begin(L);
  if (stream16) {
    FNO_DISPATCH_T(dtype, {
      if (in_ch == 2)
        k_lift_bwd16<T, 2><<<grid, LB_THREADS, 0, L.stream>>>((const T *)a, (const T *)dv, partial,
                                                              g.B, g.N, width, ncg);
      else if (in_ch == 3)
        k_lift_bwd16<T, 3><<<grid, LB_THREADS, 0, L.stream>>>((const T *)a, (const T *)dv, partial,
                                                              g.B, g.N, width, ncg);
      else
        k_lift_bwd16<T, 4><<<grid, LB_THREADS, 0, L.stream>>>((const T *)a, (const T *)dv, partial,
                                                              g.B, g.N, width, ncg);
    });
  } else {
    FNO_DISPATCH_T(dtype, k_lift_bwd<T><<<grid, PB, 0, L.stream>>>((const T *)a, (const T *)dv,
                                                                   partial, g.B, g.N, in_ch,
                                                                   width));
  }
  launch_end(L, "lift_bwd");
  return cudaGetLastError();
}

cudaError_t launch_mse(const Launch &L, long long n, int dtype, const void *u, const void *t,
                       float *loss, void *du) {
  cudaError_t err = cudaMemsetAsync(loss, 0, sizeof(float), L.stream);
  if (err != cudaSuccess) return err;
  long long want = (n + 255) / 256;
  const int grid = (int)(want < 4LL * L.num_sms ? (want > 0 ? want : 1) : 4LL * L.num_sms);
  launch_begin(L);
  FNO_DISPATCH_T(dtype, k_mse<T><<<grid, 256, 0, L.stream>>>((const T *)u, (const T *)t, loss,
                                                             (T *)du, n));
  launch_end(L, "mse");
  return cudaGetLastError();
}

}  // namespace fno
