// Truncated inverse transform of the slab and last axes with the block's
// pointwise epilogue fused in (step S4 forward, and the spectral / skip /
// weight-gradient epilogue of the backward, step S6).
//
// One thread owns one grid point and all channels of it.  A tile of
// consecutive points first expands the spectrum along the slab axis for the
// rows it touches (shared memory), then every thread sums the last-axis
// modes for its point, adds W x + b, applies GELU and writes the output: x is
// read once and y written once, each fully coalesced across the warp.
#include "fno_common.cuh"
#include "fno_kernels.cuh"

namespace fno {

namespace {

constexpr int EP_FWD_PTS = 256;
constexpr int EP_BWD_PTS = 128;
constexpr int EP_BATCH = 8;   // 16-byte loads a thread keeps in flight per array

// the 16 / sizeof(T) storage elements of a 16-byte chunk, as floats
template <typename T> __device__ __forceinline__ void unpack16(const uint4 &v, float *f);
template <> __device__ __forceinline__ void unpack16<float>(const uint4 &v, float *f) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4 &v, float *f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
template <> __device__ __forceinline__ void unpack16<__half>(const uint4 &v, float *f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __half2 h;
    memcpy(&h, &w[i], 4);
    const float2 t = __half22float2(h);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

__host__ __device__ inline size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

struct EpiLayout {
  size_t twL, twS, U, W, bias, dz, xs, acc, total;
  int maxr, Csp, Wld;
};

__host__ __device__ inline EpiLayout epi_layout(const Geom &g, int mode, int Ci, int Co,
                                                 int pts) {
  EpiLayout l;
  const int Cs = (mode <= EPI_BLOCK_FWD) ? Co : Ci;
  l.Csp = (Cs + 1) & ~1;
  l.maxr = g.S < pts / g.NL + 2 ? g.S : pts / g.NL + 2;
  size_t off = 0;
  l.twL = off;
  off = align16(off + sizeof(float2) * g.NL);
  l.twS = off;
  off = align16(off + sizeof(float2) * g.S);
  l.U = off;
  off = align16(off + sizeof(float2) * (size_t)l.maxr * g.mL * l.Csp);
  // forward: W transposed [Ci][Co pad 4]; backward: W [Co][Ci pad 4]
  l.Wld = (mode == EPI_BLOCK_BWD) ? ((Ci + 3) & ~3) : ((Co + 3) & ~3);
  l.W = off;
  if (mode == EPI_BLOCK_FWD) off = align16(off + sizeof(float) * (size_t)Ci * l.Wld);
  if (mode == EPI_BLOCK_BWD) off = align16(off + sizeof(float) * (size_t)Co * l.Wld);
  l.bias = off;
  if (mode == EPI_BLOCK_FWD) off = align16(off + sizeof(float) * Co);
  l.dz = off;
  l.xs = off;
  l.acc = off;
  if (mode == EPI_BLOCK_BWD) {   // dz and x of the tile, rows padded to pts + 1
    off = align16(off + sizeof(float) * (size_t)Co * (pts + 1));
    l.xs = off;
    off = align16(off + sizeof(float) * (size_t)(Ci + 1) * (pts + 1));
    l.acc = off;
  }
  l.total = off;
  return l;
}

template <typename T, int MODE, int CMAX, int PTS>
__global__ void __launch_bounds__(PTS) k_epilogue(EpiArgs a, Geom g) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int Ci = a.Ci, Co = a.Co;
  const EpiLayout lay = epi_layout(g, MODE, Ci, Co, PTS);
  float2 *twL = reinterpret_cast<float2 *>(smem + lay.twL);
  float2 *twS = reinterpret_cast<float2 *>(smem + lay.twS);
  float2 *U = reinterpret_cast<float2 *>(smem + lay.U);
  float *Wsm = reinterpret_cast<float *>(smem + lay.W);
  float *bias_s = reinterpret_cast<float *>(smem + lay.bias);
  float *dz_s = reinterpret_cast<float *>(smem + lay.dz);
  float *x_s = reinterpret_cast<float *>(smem + lay.xs);

  const int tid = threadIdx.x;
  const int Cs = (MODE <= EPI_BLOCK_FWD) ? Co : Ci;
  const int Csp = lay.Csp;
  const int NL = g.NL, S = g.S, mL = g.mL, QS = g.QS, O = g.O;
  const long long SN = (long long)S * NL;
  const int tiles_per_slab = (int)((SN + PTS - 1) / PTS);
  const long long ntiles = g.B * O * tiles_per_slab;
  const T *x = reinterpret_cast<const T *>(a.x);
  T *out = reinterpret_cast<T *>(a.out);

  build_twiddles(twL, NL);
  build_twiddles(twS, S);
  if (MODE == EPI_BLOCK_FWD) {
    const T *W = reinterpret_cast<const T *>(a.W);
    for (int e = tid; e < Ci * lay.Wld; e += PTS) {
      const int i = e / lay.Wld, o = e - i * lay.Wld;
      Wsm[e] = o < Co ? to_f<T>(W[o * Ci + i]) : 0.f;
    }
    const T *bias = reinterpret_cast<const T *>(a.bias);
    for (int o = tid; o < Co; o += PTS) bias_s[o] = bias ? to_f<T>(bias[o]) : 0.f;
  }
  if (MODE == EPI_BLOCK_BWD) {
    const T *W = reinterpret_cast<const T *>(a.W);
    for (int e = tid; e < Co * lay.Wld; e += PTS) {
      const int o = e / lay.Wld, i = e - o * lay.Wld;
      Wsm[e] = i < Ci ? to_f<T>(W[o * Ci + i]) : 0.f;
    }
  }
  // block backward: this thread's share of dW (a 4 x 8 block of [Co][Ci]) and
  // of db (row tid), accumulated in registers over all of the CTA's tiles
  constexpr int OB = 4, IB = 8;
  const int nib = (Ci + IB - 1) / IB;
  const int nblk = ((Co + OB - 1) / OB) * nib;
  const int ob = tid / (nib > 0 ? nib : 1), ib = tid - ob * (nib > 0 ? nib : 1);
  float accw[OB][IB];
  float accb = 0.f;
#pragma unroll
  for (int k = 0; k < OB; ++k)
#pragma unroll
    for (int m = 0; m < IB; ++m) accw[k][m] = 0.f;

  // 16-byte vector loads: aligned bases and rows whose length is a multiple of
  // the chunk (every chunk then lies wholly inside or wholly past the end)
  const bool u_vec = a.U != nullptr && mL % 2 == 0 &&
                     (reinterpret_cast<uintptr_t>(a.U) & 15) == 0;
  const bool io_vec = MODE == EPI_BLOCK_BWD && SN % (16 / (int)sizeof(T)) == 0 &&
                      ((reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.dy) |
                        (a.act ? reinterpret_cast<uintptr_t>(a.pre) : 0)) & 15) == 0;

  for (long long tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const long long slab = tile / tiles_per_slab;
    const long long p0 = (tile - slab * tiles_per_slab) * (long long)PTS;
    const long long b = slab / O;
    const int outer = (int)(slab - b * O);
    const int r_first = (int)(p0 / NL);
    const int r_last = (int)min((long long)S - 1, (p0 + PTS - 1) / NL);
    const int nr = r_last - r_first + 1;
    __syncthreads();  // previous tile is done with U / dz_s / x_s
    // slab-axis inverse for the rows of this tile: U[row][k][c]
    if (u_vec) {
      // precomputed slab inverse: the tile's rows of one channel are nr * mL
      // consecutive values; 16-byte chunks (two modes), a batch in flight
      const int h = nr * mL / 2, nu = Cs * h;
      for (int e0 = tid; e0 < nu; e0 += EP_BATCH * PTS) {
        float4 v[EP_BATCH];
#pragma unroll
        for (int m = 0; m < EP_BATCH; ++m) {
          const int e = e0 + m * PTS;
          if (e < nu) {
            const int c = e / h, kk = e - c * h;
            const float4 *src = reinterpret_cast<const float4 *>(
                a.U + (((b * Cs + c) * O + outer) * (long long)S + r_first) * mL);
            v[m] = __ldg(src + kk);
          }
        }
#pragma unroll
        for (int m = 0; m < EP_BATCH; ++m) {
          const int e = e0 + m * PTS;
          if (e < nu) {
            const int c = e / h, kk = e - c * h;
            U[(2 * kk) * Csp + c] = make_float2(v[m].x, v[m].y);
            U[(2 * kk + 1) * Csp + c] = make_float2(v[m].z, v[m].w);
          }
        }
      }
    } else
    for (int e = tid; e < nr * mL * Cs; e += PTS) {
      const int k = e % mL;
      const int rest = e / mL;
      const int rl = rest % nr, c = rest / nr;
      const int row = r_first + rl;
      const float2 *z = a.Z + (((b * Cs + c) * O + outer) * QS) * (long long)mL + k;
      float2 s = make_float2(0.f, 0.f);
      if (a.U) {   // precomputed slab inverse
        s = a.U[(((b * Cs + c) * O + outer) * (long long)S + row) * mL + k];
      } else {
        KeptIndex ki(QS == 1 ? 0 : g.mS, S, row);
        for (int q = 0; q < QS; ++q) cfma(s, __ldg(z + (long long)q * mL), twS[ki.next()]);
      }
      U[(rl * mL + k) * Csp + c] = s;
    }
    if (Cs & 1)
      for (int e = tid; e < nr * mL; e += PTS) U[e * Csp + Cs] = make_float2(0.f, 0.f);

    const long long pt = p0 + tid;
    const bool valid = pt < SN;
    const long long base_o = (b * Co * O + outer) * SN + pt;  // + o * O * SN
    const long long base_i = (b * Ci * O + outer) * SN + pt;  // + i * O * SN
    const long long cstride = (long long)O * SN;
    if (MODE == EPI_BLOCK_BWD && io_vec) {
      // dz = dy * GELU'(pre) and x of the tile from 16-byte chunks of VEC
      // consecutive points of one channel; a batch of chunks of all three
      // arrays in flight per thread, points past the end read as zeros
      constexpr int VEC = 16 / sizeof(T), CPR = PTS / VEC;
      const T *dy = reinterpret_cast<const T *>(a.dy);
      const T *pre = reinterpret_cast<const T *>(a.pre);
      const int ndz = Co * CPR, nxc = Ci * CPR, nmax = ndz > nxc ? ndz : nxc;
      const long long bo = (b * Co * O + outer) * SN + p0, bi = (b * Ci * O + outer) * SN + p0;
      for (int c0 = tid; c0 < nmax; c0 += EP_BATCH * PTS) {
        uint4 vd[EP_BATCH], vp[EP_BATCH], vx[EP_BATCH];
#pragma unroll
        for (int m = 0; m < EP_BATCH; ++m) {
          const int c = c0 + m * PTS;
          const int row = c / CPR, q = c - row * CPR;
          const bool in = p0 + q * VEC < SN;
          vd[m] = vp[m] = vx[m] = make_uint4(0u, 0u, 0u, 0u);
          if (in && c < ndz) {
            const long long off = bo + row * cstride + q * VEC;
            vd[m] = __ldg(reinterpret_cast<const uint4 *>(dy + off));
            if (a.act) vp[m] = __ldg(reinterpret_cast<const uint4 *>(pre + off));
          }
          if (in && c < nxc)
            vx[m] = __ldg(reinterpret_cast<const uint4 *>(x + bi + row * cstride + q * VEC));
        }
#pragma unroll
        for (int m = 0; m < EP_BATCH; ++m) {
          const int c = c0 + m * PTS;
          const int row = c / CPR, q = c - row * CPR;
          if (c < ndz) {
            float d[VEC], pv[VEC];
            unpack16<T>(vd[m], d);
            unpack16<T>(vp[m], pv);
            float *dst = dz_s + row * (PTS + 1) + q * VEC;
#pragma unroll
            for (int i = 0; i < VEC; ++i) dst[i] = a.act ? d[i] * gelu_grad_f(pv[i]) : d[i];
          }
          if (c < nxc) {
            float xv[VEC];
            unpack16<T>(vx[m], xv);
            float *dst = x_s + row * (PTS + 1) + q * VEC;
#pragma unroll
            for (int i = 0; i < VEC; ++i) dst[i] = xv[i];
          }
        }
      }
    } else if (MODE == EPI_BLOCK_BWD) {
      const T *dy = reinterpret_cast<const T *>(a.dy);
      const T *pre = reinterpret_cast<const T *>(a.pre);
      for (int o = 0; o < Co; ++o) {
        float dz = 0.f;
        if (valid) {
          const float d = ldf<T>(dy + base_o + o * cstride);
          dz = a.act ? d * gelu_grad_f(ldf<T>(pre + base_o + o * cstride)) : d;
        }
        dz_s[o * (PTS + 1) + tid] = dz;
      }
      for (int i = 0; i < Ci; ++i)
        x_s[i * (PTS + 1) + tid] = valid ? ldf<T>(x + base_i + i * cstride) : 0.f;
      x_s[Ci * (PTS + 1) + tid] = valid ? 1.f : 0.f;
    }
    __syncthreads();

    if (valid) {
      const int r = (int)(pt / NL);
      const int n = (int)(pt - (long long)r * NL);
      const int rl = r - r_first;
      float u[CMAX];
#pragma unroll
      for (int c = 0; c < CMAX; ++c) u[c] = 0.f;
      int idx = 0;
      for (int k = 0; k < mL; ++k) {
        const float2 w = twL[idx];
        idx += n;
        if (idx >= NL) idx -= NL;
        const float4 *up = reinterpret_cast<const float4 *>(U + (rl * mL + k) * Csp);
#pragma unroll
        for (int c2 = 0; c2 < CMAX / 2; ++c2) {
          if (2 * c2 < Cs) {
            const float4 v = up[c2];
            u[2 * c2] = fmaf(v.x, w.x, fmaf(-v.y, w.y, u[2 * c2]));
            u[2 * c2 + 1] = fmaf(v.z, w.x, fmaf(-v.w, w.y, u[2 * c2 + 1]));
          }
        }
      }
      if (MODE == EPI_SPEC) {
#pragma unroll
        for (int o = 0; o < CMAX; ++o)
          if (o < Co) out[base_o + o * cstride] = from_f<T>(u[o]);
      } else if (MODE == EPI_BLOCK_FWD) {
#pragma unroll
        for (int o = 0; o < CMAX; ++o)
          if (o < Co) u[o] += bias_s[o];
        for (int i = 0; i < Ci; ++i) {
          const float xi = ldf<T>(x + base_i + i * cstride);
          const float4 *wp = reinterpret_cast<const float4 *>(Wsm + i * lay.Wld);
#pragma unroll
          for (int o4 = 0; o4 < CMAX / 4; ++o4) {
            if (4 * o4 < Co) {
              const float4 w = wp[o4];
              u[4 * o4] = fmaf(w.x, xi, u[4 * o4]);
              u[4 * o4 + 1] = fmaf(w.y, xi, u[4 * o4 + 1]);
              u[4 * o4 + 2] = fmaf(w.z, xi, u[4 * o4 + 2]);
              u[4 * o4 + 3] = fmaf(w.w, xi, u[4 * o4 + 3]);
            }
          }
        }
        T *pre_out = reinterpret_cast<T *>(a.pre_out);
#pragma unroll
        for (int o = 0; o < CMAX; ++o) {
          if (o < Co) {
            const float p = u[o];
            if (pre_out) pre_out[base_o + o * cstride] = from_f<T>(p);
            out[base_o + o * cstride] = from_f<T>(a.act ? gelu_f(p) : p);
          }
        }
      } else if (MODE == EPI_SPEC_BWD) {
#pragma unroll
        for (int i = 0; i < CMAX; ++i) {
          if (i < Ci) {
            float v = u[i];
            if (a.tanh_pre) {
              const float t = tanhf(ldf<T>(x + base_i + i * cstride));
              v *= 1.f - t * t;
            }
            out[base_i + i * cstride] = from_f<T>(v);
          }
        }
      } else {  // EPI_BLOCK_BWD
        if (a.tanh_pre) {
#pragma unroll
          for (int i = 0; i < CMAX; ++i) {
            if (i < Ci) {
              const float t = tanhf(x_s[i * (PTS + 1) + tid]);
              u[i] *= 1.f - t * t;
            }
          }
        }
        for (int o = 0; o < Co; ++o) {
          const float dzo = dz_s[o * (PTS + 1) + tid];
          const float4 *wp = reinterpret_cast<const float4 *>(Wsm + o * lay.Wld);
#pragma unroll
          for (int i4 = 0; i4 < CMAX / 4; ++i4) {
            if (4 * i4 < Ci) {
              const float4 w = wp[i4];
              u[4 * i4] = fmaf(w.x, dzo, u[4 * i4]);
              u[4 * i4 + 1] = fmaf(w.y, dzo, u[4 * i4 + 1]);
              u[4 * i4 + 2] = fmaf(w.z, dzo, u[4 * i4 + 2]);
              u[4 * i4 + 3] = fmaf(w.w, dzo, u[4 * i4 + 3]);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < CMAX; ++i)
          if (i < Ci) out[base_i + i * cstride] = from_f<T>(u[i]);
      }
    }
    if (MODE == EPI_BLOCK_BWD) {
      // dW[o][i] += sum_p dz[o][p] x[i][p] over this tile's points (4 x 8
      // outer products per point from shared memory), db[o] += sum_p dz[o][p]
      if (tid < nblk) {
        for (int pp = 0; pp < PTS; ++pp) {
          float dzv[OB], xv[IB];
#pragma unroll
          for (int k = 0; k < OB; ++k)
            dzv[k] = ob * OB + k < Co ? dz_s[(ob * OB + k) * (PTS + 1) + pp] : 0.f;
#pragma unroll
          for (int m = 0; m < IB; ++m)
            xv[m] = ib * IB + m < Ci ? x_s[(ib * IB + m) * (PTS + 1) + pp] : 0.f;
#pragma unroll
          for (int k = 0; k < OB; ++k)
#pragma unroll
            for (int m = 0; m < IB; ++m) accw[k][m] = fmaf(dzv[k], xv[m], accw[k][m]);
        }
      }
      if (tid < Co) {
        const float *dzr = dz_s + tid * (PTS + 1);
        for (int pp = 0; pp < PTS; ++pp) accb += dzr[pp];
      }
    }
  }
  if (MODE == EPI_BLOCK_BWD) {
    float *dst = a.partial + (long long)blockIdx.x * Co * (Ci + 1);
    if (tid < nblk) {
#pragma unroll
      for (int k = 0; k < OB; ++k)
#pragma unroll
        for (int m = 0; m < IB; ++m) {
          const int o = ob * OB + k, i = ib * IB + m;
          if (o < Co && i < Ci) dst[o * (Ci + 1) + i] = accw[k][m];
        }
    }
    if (tid < Co) dst[tid * (Ci + 1) + Ci] = accb;
  }
}

template <typename T, int MODE, int CMAX>
cudaError_t launch_epi_t(const Launch &L, const Geom &g, const EpiArgs &a) {
  constexpr int PTS = MODE == EPI_BLOCK_BWD ? EP_BWD_PTS : EP_FWD_PTS;
  const EpiLayout lay = epi_layout(g, MODE, a.Ci, a.Co, PTS);
  const int grid = epi_grid(g, MODE, L.num_sms);
  auto kern = k_epilogue<T, MODE, CMAX, PTS>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.total);
  static const char *const tags[4] = {"epi_spec", "epi_block_fwd", "epi_spec_bwd",
                                      "epi_block_bwd"};
  launch_begin(L);
  kern<<<grid, PTS, lay.total, L.stream>>>(a, g);
  launch_end(L, tags[MODE]);
  return cudaGetLastError();
}

template <typename T, int MODE>
cudaError_t launch_epi_c(const Launch &L, const Geom &g, const EpiArgs &a) {
  const int c = a.Ci > a.Co ? a.Ci : a.Co;
  if (c <= 16) return launch_epi_t<T, MODE, 16>(L, g, a);
  if (c <= 32) return launch_epi_t<T, MODE, 32>(L, g, a);
  return launch_epi_t<T, MODE, 64>(L, g, a);
}

template <typename T>
cudaError_t launch_epi_m(const Launch &L, const Geom &g, int mode, const EpiArgs &a) {
  switch (mode) {
    case EPI_SPEC: return launch_epi_c<T, EPI_SPEC>(L, g, a);
    case EPI_BLOCK_FWD: return launch_epi_c<T, EPI_BLOCK_FWD>(L, g, a);
    case EPI_SPEC_BWD: return launch_epi_c<T, EPI_SPEC_BWD>(L, g, a);
    default: return launch_epi_c<T, EPI_BLOCK_BWD>(L, g, a);
  }
}

// Sum of the per-CTA partial rows: a CTA takes 32 columns, its eight warps
// the parts w, w + 8, ... of them (eight loads in flight per thread), and the
// eight part sums meet in shared memory in a fixed order.
constexpr int RP_COLS = 32, RP_SLICES = 8;
__global__ void __launch_bounds__(RP_COLS * RP_SLICES)
    k_reduce_partials(const float *__restrict__ partial, int nparts, long long stride,
                      long long offset, int rows, int cols, float *__restrict__ out_main,
                      float *__restrict__ out_last) {
  __shared__ float part[RP_SLICES][RP_COLS];
  const int lane = threadIdx.x & 31, sl = threadIdx.x >> 5;
  const int e = blockIdx.x * RP_COLS + lane;
  const bool in = e < rows * (cols + 1);
  float s = 0.f;
  if (in) {
    const float *src = partial + offset + e;
#pragma unroll 8
    for (int p = sl; p < nparts; p += RP_SLICES) s += src[p * stride];
  }
  part[sl][lane] = s;
  __syncthreads();
  if (sl != 0 || !in) return;
  float t = part[0][lane];
#pragma unroll
  for (int i = 1; i < RP_SLICES; ++i) t += part[i][lane];
  const int r = e / (cols + 1), c = e - r * (cols + 1);
  if (c < cols) {
    if (out_main) out_main[r * cols + c] = t;
  } else if (out_last) {
    out_last[r] = t;
  }
}

}  // namespace

size_t epi_smem_bytes(const Geom &g, int mode, int Ci, int Co) {
  const int pts = mode == EPI_BLOCK_BWD ? EP_BWD_PTS : EP_FWD_PTS;
  return epi_layout(g, mode, Ci, Co, pts).total;
}

int epi_grid(const Geom &g, int mode, int num_sms) {
  const int pts = mode == EPI_BLOCK_BWD ? EP_BWD_PTS : EP_FWD_PTS;
  const long long SN = (long long)g.S * g.NL;
  const long long ntiles = g.B * g.O * ((SN + pts - 1) / pts);
  const long long cap = mode == EPI_BLOCK_BWD ? (long long)kPartialCTAs : (long long)num_sms * 8;
  return (int)(ntiles < cap ? ntiles : cap);
}

size_t epi_partial_bytes(const Geom &g, int Ci, int Co, int num_sms) {
  return sizeof(float) * (size_t)epi_grid(g, EPI_BLOCK_BWD, num_sms) * Co * (Ci + 1);
}

cudaError_t launch_epilogue(const Launch &L, const Geom &g, int dtype, int mode,
                            const EpiArgs &a) {
  if (dtype == DT_F32) return launch_epi_m<float>(L, g, mode, a);
  if (dtype == DT_F16) return launch_epi_m<__half>(L, g, mode, a);
  return launch_epi_m<__nv_bfloat16>(L, g, mode, a);
}

cudaError_t launch_reduce_rows(const Launch &L, const float *partial, int nparts,
                               long long stride, long long offset, int rows, int cols,
                               float *out_main, float *out_last) {
  const int n = rows * (cols + 1);
  launch_begin(L);
  k_reduce_partials<<<(n + RP_COLS - 1) / RP_COLS, RP_COLS * RP_SLICES, 0, L.stream>>>(
      partial, nparts, stride, offset, rows, cols, out_main, out_last);
  launch_end(L, "reduce_partials");
  return cudaGetLastError();
}

}  // namespace fno
