// C ABI of the FNO library (include/fno.h): argument validation, workspace
// layout and the launch sequence of each operation.  All arithmetic runs in
// the kernels of transform.cu, mix.cu, epilogue.cu and net.cu.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "fno.h"
#include "fno_kernels.cuh"
#include "tc_util.cuh"

using namespace fno;

namespace {

thread_local char g_err[512] = "";
thread_local int g_launches = 0;
int g_use_tc = 1;   // tensor-core kernels where the shape allows (fno_set_tensor_cores)

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char *where) {
  return fail(FNO_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

#define FNO_TRY(expr, where)                       \
  do {                                             \
    cudaError_t _e = (expr);                       \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

constexpr size_t kSmemLimit = 227 * 1024;

size_t elsize(int dtype) { return dtype == FNO_F32 ? 4 : 2; }
size_t al(size_t v) { return (v + 255) & ~(size_t)255; }
bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

int device_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
    return n;
  cudaGetLastError();
  return 148;
}

// Build the flattened geometry; returns FNO_OK or an error code (message set).
int make_geom(int ndim, int64_t batch, const int64_t *grid, const int *modes, Geom *g) {
  if (ndim < 1 || ndim > FNO_MAX_DIMS) return fail(FNO_ERR_INVALID_ARG, "ndim %d not in 1..3", ndim);
  if (batch < 1) return fail(FNO_ERR_INVALID_ARG, "batch %lld < 1", (long long)batch);
  for (int j = 0; j < ndim; ++j) {
    if (grid[j] < 1) return fail(FNO_ERR_INVALID_ARG, "grid[%d] = %lld < 1", j, (long long)grid[j]);
    if (grid[j] > kMaxAxis)
      return fail(FNO_ERR_UNSUPPORTED, "grid[%d] = %lld exceeds %d", j, (long long)grid[j], kMaxAxis);
    if (j < ndim - 1) {
      if (modes[j] < 1 || 2LL * modes[j] > grid[j])
        return fail(FNO_ERR_INVALID_ARG, "modes[%d] = %d: need 1 <= 2 modes <= grid (%lld)", j,
                    modes[j], (long long)grid[j]);
    } else {
      if (modes[j] < 1 || modes[j] > grid[j] / 2 + 1)
        return fail(FNO_ERR_INVALID_ARG, "modes[%d] = %d: need 1 <= modes <= grid/2 + 1 (%lld)", j,
                    modes[j], (long long)grid[j]);
      if (modes[j] > 64) return fail(FNO_ERR_UNSUPPORTED, "last-axis modes %d > 64", modes[j]);
    }
  }
  Geom x{};
  x.d = ndim;
  x.B = batch;
  x.NL = (int)grid[ndim - 1];
  x.mL = modes[ndim - 1];
  if (ndim >= 2) {
    x.S = (int)grid[ndim - 2];
    x.mS = modes[ndim - 2];
    x.QS = 2 * x.mS;
  } else {
    x.S = 1; x.mS = 0; x.QS = 1;
  }
  if (ndim == 3) {
    x.O = (int)grid[0];
    x.mO = modes[0];
    x.QO = 2 * x.mO;
  } else {
    x.O = 1; x.mO = 0; x.QO = 1;
  }
  x.N = (long long)x.O * x.S * x.NL;
  x.K = (long long)x.QO * x.QS * x.mL;
  x.inv_n = (float)(1.0 / (double)x.N);
  *g = x;
  return FNO_OK;
}

int check_block(const fno_block_desc *d, Geom *g) {
  if (!d) return fail(FNO_ERR_INVALID_ARG, "descriptor is NULL");
  if (d->dtype < FNO_F32 || d->dtype > FNO_BF16)
    return fail(FNO_ERR_INVALID_ARG, "dtype %d unknown", d->dtype);
  if (d->flags & ~(unsigned)(FNO_TANH_PREACT | FNO_NO_ACT))
    return fail(FNO_ERR_INVALID_ARG, "unknown flag bits 0x%x", d->flags);
  if (d->cin < 1 || d->cout < 1)
    return fail(FNO_ERR_INVALID_ARG, "channels cin=%d cout=%d must be >= 1", d->cin, d->cout);
  if (d->cin > kMaxWidth || d->cout > kMaxWidth)
    return fail(FNO_ERR_UNSUPPORTED, "channels cin=%d cout=%d exceed %d", d->cin, d->cout,
                kMaxWidth);
  int rc = make_geom(d->ndim, d->batch, d->grid, d->modes, g);
  if (rc) return rc;
  return FNO_OK;
}

// Workspace map of a block operation.
struct BlockWs {
  size_t zpart, xhat, yhat, zexp, u, img, dxhat, partial, rcp, drcp, cps, total;
};

BlockWs block_ws(const Geom &g, int Ci, int Co, int op) {
  BlockWs w{};
  const size_t cplx = sizeof(float2);
  const long long Cmax = Ci > Co ? Ci : Co;
  size_t off = 0;
  w.zpart = off;  // forward transform of Ci channels (x) and of Co channels (dz)
  {
    const size_t zi = fwd_zpart_bytes(g, Ci), zo = fwd_zpart_bytes(g, Co);
    off += al(zi > zo ? zi : zo);
  }
  w.xhat = off;                       // used when the caller gives no xhat buffer
  off += al(cplx * (size_t)(g.B * Ci * g.K));
  w.yhat = off;                       // yhat (forward) or D = DFT_K(dz) (backward)
  off += al(cplx * (size_t)(g.B * Cmax * g.K));
  w.zexp = off;
  off += al(inv_expand_bytes(g, Cmax));
  w.u = off;                          // spectrum inverted along the slab axis
  off += al(inv_slab_bytes(g, Cmax));
  w.img = off;                        // or, per grid row, the epilogue's B operand image
  if (op == FNO_OP_SPECTRAL_FWD || op == FNO_OP_BLOCK_FWD)
    off += al(g.d == 2 ? (size_t)g.B * g.S * epi_img_row_bytes(DT_F32, Co, g.mL) : 0);
  w.dxhat = off;
  w.partial = off;
  const bool cp = op == FNO_OP_SPECTRAL_BWD_CP || op == FNO_OP_BLOCK_BWD_CP;
  const bool bwd = op == FNO_OP_SPECTRAL_BWD || op == FNO_OP_BLOCK_BWD || cp;
  const bool block_bwd = op == FNO_OP_BLOCK_BWD || op == FNO_OP_BLOCK_BWD_CP;
  if (bwd) {
    off += al(cplx * (size_t)(g.B * Ci * g.K));
    w.partial = off;
    if (block_bwd) off += al(sizeof(float) * (size_t)kPartialCTAs * Co * (Ci + 1));
  }
  w.rcp = w.drcp = w.cps = off;
  if (cp) {   // the rebuilt weight (float32-sized), its gradient, the projection scratch
    w.rcp = off;
    off += al(sizeof(float2) * (size_t)Ci * Co * g.K);
    w.drcp = off;
    off += al(sizeof(float2) * (size_t)Ci * Co * g.K);
    w.cps = off;
    off += al(sizeof(float2) * (size_t)Ci * kMaxCpRank);
  }
  w.total = off;
  return w;
}

int check_smem(const Geom &g, int Ci, int Co, int op) {
  const int epi_mode = op == FNO_OP_SPECTRAL_FWD   ? EPI_SPEC
                       : op == FNO_OP_BLOCK_FWD    ? EPI_BLOCK_FWD
                       : op == FNO_OP_SPECTRAL_BWD ? EPI_SPEC_BWD
                                                   : EPI_BLOCK_BWD;
  const size_t e = epi_smem_bytes(g, epi_mode, Ci, Co);
  if (e > kSmemLimit)
    return fail(FNO_ERR_UNSUPPORTED, "epilogue needs %zu B of shared memory (> %zu)", e, kSmemLimit);
  const size_t f = sizeof(float2) * ((size_t)g.NL + g.S + 64 * (size_t)g.mL * 2 + (size_t)g.QS * g.mL) +
                   sizeof(float) * 64 * 65;
  if (f > kSmemLimit)
    return fail(FNO_ERR_UNSUPPORTED, "forward transform needs %zu B of shared memory", f);
  return FNO_OK;
}

// ---------------------------------------------------------------------------
// per-kernel timing (fno_profile_*)
// ---------------------------------------------------------------------------
struct ProfRec {
  cudaEvent_t start, stop;
  const char *tag;
};
std::mutex g_prof_mu;
std::vector<ProfRec> g_prof;   // event pool; the first g_prof_used entries are live
size_t g_prof_used = 0;
bool g_prof_on = false;

// [0]: set by kernels whose bounded waits expire; [1]: the wait limit they use
// (suspended polls per wait, fno_set_wait_limit)
__device__ int g_fno_device_error[2] = {0, FNO_DEFAULT_WAIT_SPINS};

std::mutex g_err_word_mu;

int *device_error_word() {
  static int *addr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_err_word_mu);   // first calls may race from several threads
  if (!addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fno_device_error) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<int *>(p);
  }
  return addr[dev];
}

Launch make_launch(fno_stream_t s) {
  g_launches = 0;
  Launch L{reinterpret_cast<cudaStream_t>(s), &g_launches, device_sms(), g_use_tc,
           device_error_word()};
  return L;
}

// The slab-axis inverse U = E_S Z: the pruned FFT on the default paths where
// the shape allows it, else the dense sum.
cudaError_t invert_slab(const Launch &L, const Geom &g, long long C, const float2 *Z, float2 *U) {
  if ((L.tc == 1 || L.tc == 4) && inv_slab_fft_supported(g))
    return launch_inv_slab_fft(L, g, C, Z, U);
  return launch_inv_slab(L, g, C, Z, U);
}

// u_ready: U (ws + w.u) already holds the spectrum inverted along the slab
// axis (launch_spec_mid), so no slab-axis inverse is launched here.
// nparts (block backward): the number of per-CTA dW / db partials written
cudaError_t run_epilogue(const Launch &L, const Geom &g, int dtype, int mode, const EpiArgs &a,
                         unsigned char *ws, const BlockWs &w, bool u_ready = false,
                         int *nparts = nullptr) {
  float2 *U = reinterpret_cast<float2 *>(ws + w.u);
  // channels of the spectrum being inverted: Ci for the backward modes (dxhat)
  const int cs = (mode == EPI_SPEC_BWD || mode == EPI_BLOCK_BWD) ? a.Ci : a.Co;
  if (nparts) *nparts = epi_grid(g, EPI_BLOCK_BWD, L.num_sms);
  if (mode == EPI_BLOCK_BWD && nparts && (L.tc == 1 || L.tc == 3 || L.tc == 4) &&
      epi_bwd_pipe_supported(g, dtype, a.Ci, a.Co, a.tanh_pre, a.x, a.dy, a.pre, a.act, U)) {
    if (!u_ready) {
      cudaError_t e = invert_slab(L, g, cs, a.Z, U);
      if (e != cudaSuccess) return e;
    }
    return launch_epi_bwd_pipe(L, g, dtype, a, U, nparts);
  }
  if ((L.tc == 1 || L.tc == 3 || L.tc == 4) && epi_pipe_supported(g, dtype, mode, a.Ci, a.Co, a.x, U)) {
    if (!u_ready) {
      cudaError_t e = invert_slab(L, g, cs, a.Z, U);
      if (e != cudaSuccess) return e;
    }
    return launch_epi_pipe(L, g, dtype, mode, a, U);
  }
  if (L.tc && epi_tc_supported(g, dtype, mode, a.Ci, a.Co)) {
    if (!u_ready) {
      cudaError_t e = invert_slab(L, g, cs, a.Z, U);
      if (e != cudaSuccess) return e;
    }
    return launch_epilogue_tc(L, g, dtype, mode, a, U);
  }
  if (u_ready) {
    EpiArgs b = a;
    b.U = U;
    return launch_epilogue(L, g, dtype, mode, b);
  }
  if (mode == EPI_BLOCK_BWD && g.S > 1) {
    // the block backward reads the slab-axis inverse once per row instead of
    // recomputing it in every tile
    cudaError_t e = invert_slab(L, g, cs, a.Z, U);
    if (e != cudaSuccess) return e;
    EpiArgs b = a;
    b.U = U;
    return launch_epilogue(L, g, dtype, mode, b);
  }
  return launch_epilogue(L, g, dtype, mode, a);
}

// ---------------------------------------------------------------------------
// block-level building blocks (validated arguments)
// ---------------------------------------------------------------------------

// cp (optional): CP-factorised weights of the given rank in place of R
int run_forward(const Launch &L, const Geom &g, int dtype, unsigned flags, int Ci, int Co,
                const void *x, const void *R, const void *W, const void *b, void *y, void *pre,
                float *xhat_save, unsigned char *ws, int epi_mode, const CpFactors *cp = nullptr,
                int rank = 0) {
  const BlockWs w = block_ws(g, Ci, Co, epi_mode == EPI_SPEC ? FNO_OP_SPECTRAL_FWD : FNO_OP_BLOCK_FWD);
  float2 *zpart = reinterpret_cast<float2 *>(ws + w.zpart);
  float2 *xhat = xhat_save ? reinterpret_cast<float2 *>(xhat_save)
                           : reinterpret_cast<float2 *>(ws + w.xhat);
  float2 *yhat = reinterpret_cast<float2 *>(ws + w.yhat);
  FNO_TRY(launch_fwd_transform(L, g, dtype, (flags & FNO_TANH_PREACT) ? LOAD_TANH : LOAD_PLAIN,
                               Ci, x, nullptr, zpart, xhat),
          "forward transform");
  // 2D grids on the default path: mixing and the slab-axis inverse in one launch
  const bool mid = !cp && (L.tc == 1 || L.tc == 4) && spec_mid_supported(g, Ci, Co);
  // the slab-axis inverse writes the epilogue's B operand directly where the
  // pipelined epilogue takes it
  const bool img = mid && epi_img_supported(g, dtype, epi_mode, Ci, Co) &&
                   spec_mid_img_supported(g, Co) &&
                   epi_pipe_supported(g, dtype, epi_mode, Ci, Co, x, ws + w.u);
  if (cp)
    FNO_TRY(launch_mix_cp(L, g, dtype, Ci, Co, rank, xhat, *cp, yhat), "factorised mixing");
  else if (mid)
    FNO_TRY(launch_spec_mid(L, g, dtype, Ci, Co, xhat, R, yhat,
                            reinterpret_cast<float2 *>(ws + w.u), img ? ws + w.img : nullptr,
                            epi_mode == EPI_BLOCK_FWD ? b : nullptr),
            "mixing and slab-axis inverse");
  else
    FNO_TRY(launch_mix_fwd(L, g, dtype, Ci, Co, xhat, R, yhat), "mixing");
  const float2 *Z = yhat;
  if (g.QO > 1) {
    float2 *zexp = reinterpret_cast<float2 *>(ws + w.zexp);
    FNO_TRY(launch_inv_expand(L, g, Co, yhat, zexp), "outer-axis inverse");
    Z = zexp;
  }
  EpiArgs a{};
  a.Z = Z;
  a.x = x;
  a.W = W;
  a.bias = b;
  a.out = y;
  a.pre_out = pre;
  a.Ci = Ci;
  a.Co = Co;
  a.act = !(flags & FNO_NO_ACT);
  a.tanh_pre = (flags & FNO_TANH_PREACT) ? 1 : 0;
  a.img = img ? ws + w.img : nullptr;
  FNO_TRY(run_epilogue(L, g, dtype, epi_mode, a, ws, w, mid), "epilogue");
  return FNO_OK;
}

// ws_op: the operation whose workspace map `ws` follows (the dense op, or its
// factorised variant, whose map extends it)
int run_backward(const Launch &L, const Geom &g, int dtype, unsigned flags, int Ci, int Co,
                 const void *x, const float *xhat_save, const void *R, const void *W,
                 const void *pre, const void *dy, void *dx, float *dR, float *dW, float *db,
                 unsigned char *ws, bool block, int ws_op = -1) {
  const BlockWs w = block_ws(g, Ci, Co,
                             ws_op >= 0 ? ws_op : block ? FNO_OP_BLOCK_BWD : FNO_OP_SPECTRAL_BWD);
  float2 *zpart = reinterpret_cast<float2 *>(ws + w.zpart);
  const float2 *xhat = reinterpret_cast<const float2 *>(xhat_save);
  if (!xhat) {
    float2 *xh = reinterpret_cast<float2 *>(ws + w.xhat);
    FNO_TRY(launch_fwd_transform(L, g, dtype, (flags & FNO_TANH_PREACT) ? LOAD_TANH : LOAD_PLAIN,
                                 Ci, x, nullptr, zpart, xh),
            "forward transform (recompute)");
    xhat = xh;
  }
  float2 *D = reinterpret_cast<float2 *>(ws + w.yhat);
  const bool act = block && !(flags & FNO_NO_ACT);
  FNO_TRY(launch_fwd_transform(L, g, dtype, act ? LOAD_DZ : LOAD_PLAIN, Co, dy, pre, zpart, D),
          "transform of dz");
  FNO_TRY(launch_mix_bwd_dr(L, g, dtype, Ci, Co, xhat, D, dR), "dR");
  float2 *dxhat = reinterpret_cast<float2 *>(ws + w.dxhat);
  FNO_TRY(launch_mix_bwd_dx(L, g, dtype, Ci, Co, D, R, dxhat), "dxhat");
  const float2 *Z = dxhat;
  if (g.QO > 1) {
    float2 *zexp = reinterpret_cast<float2 *>(ws + w.zexp);
    FNO_TRY(launch_inv_expand(L, g, Ci, dxhat, zexp), "outer-axis inverse");
    Z = zexp;
  }
  EpiArgs a{};
  a.Z = Z;
  a.x = x;
  a.W = W;
  a.dy = dy;
  a.pre = pre;
  a.out = dx;
  a.Ci = Ci;
  a.Co = Co;
  a.act = act ? 1 : 0;
  a.tanh_pre = (flags & FNO_TANH_PREACT) ? 1 : 0;
  float *partial = reinterpret_cast<float *>(ws + w.partial);
  a.partial = partial;
  int nparts = 0;
  FNO_TRY(run_epilogue(L, g, dtype, block ? EPI_BLOCK_BWD : EPI_SPEC_BWD, a, ws, w, false,
                       &nparts),
          "epilogue");
  if (block) {
    FNO_TRY(launch_reduce_rows(L, partial, nparts, (long long)Co * (Ci + 1), 0, Co, Ci, dW, db),
            "dW/db reduction");
  }
  return FNO_OK;
}

#define REQUIRE_PTR(p, name)                                                           \
  do {                                                                                 \
    if (!(p)) return fail(FNO_ERR_INVALID_ARG, "%s is NULL", name);                    \
    if (!aligned16(p)) return fail(FNO_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)
#define OPTIONAL_PTR(p, name)                                                           \
  do {                                                                                  \
    if ((p) && !aligned16(p)) return fail(FNO_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

// ---------------------------------------------------------------------------
// network helpers
// ---------------------------------------------------------------------------

int check_net(const fno_net_desc *d, Geom *g) {
  if (!d) return fail(FNO_ERR_INVALID_ARG, "descriptor is NULL");
  if (d->dtype < FNO_F32 || d->dtype > FNO_BF16)
    return fail(FNO_ERR_INVALID_ARG, "dtype %d unknown", d->dtype);
  if (d->flags & ~(unsigned)(FNO_TANH_PREACT | FNO_NO_ACT))
    return fail(FNO_ERR_INVALID_ARG, "unknown flag bits 0x%x", d->flags);
  if (d->n_layers < 1 || d->n_layers > FNO_MAX_LAYERS)
    return fail(FNO_ERR_INVALID_ARG, "n_layers %d not in 1..%d", d->n_layers, FNO_MAX_LAYERS);
  if (d->in_channels < 1 || d->in_channels > 8)
    return fail(d->in_channels < 1 ? FNO_ERR_INVALID_ARG : FNO_ERR_UNSUPPORTED,
                "in_channels %d not in 1..8", d->in_channels);
  if (d->width < 1 || d->width > kMaxWidth)
    return fail(d->width < 1 ? FNO_ERR_INVALID_ARG : FNO_ERR_UNSUPPORTED, "width %d not in 1..%d",
                d->width, kMaxWidth);
  if (d->out_channels < 1 || d->out_channels > 4)
    return fail(d->out_channels < 1 ? FNO_ERR_INVALID_ARG : FNO_ERR_UNSUPPORTED,
                "out_channels %d not in 1..4", d->out_channels);
  if (d->hidden < 1) return fail(FNO_ERR_INVALID_ARG, "hidden %d < 1", d->hidden);
  int rc = make_geom(d->ndim, d->batch, d->grid, d->modes, g);
  if (rc) return rc;
  const size_t pb = proj_bwd_smem_bytes(d->width, d->hidden, d->out_channels);
  if (pb > kSmemLimit)
    return fail(FNO_ERR_UNSUPPORTED, "projection hidden %d too wide", d->hidden);
  return check_smem(*g, d->width, d->width, FNO_OP_BLOCK_BWD);
}

struct NetWs {
  size_t block, act0, act1, partial, total;
};

NetWs net_ws(const fno_net_desc *d, const Geom &g, int op) {
  NetWs w{};
  const size_t act = al(elsize(d->dtype) * (size_t)(g.B * d->width * g.N));
  const BlockWs bw = block_ws(g, d->width, d->width,
                              op == FNO_OP_NET_FWD ? FNO_OP_BLOCK_FWD : FNO_OP_BLOCK_BWD);
  size_t off = 0;
  w.block = off;
  off += al(bw.total);
  w.act0 = off;
  off += act;
  w.act1 = off;
  off += act;
  w.partial = off;
  if (op == FNO_OP_NET_BWD) {
    size_t p = proj_bwd_partial_floats(d->width, d->hidden, d->out_channels);
    const size_t lift = (size_t)d->width * (d->in_channels + 1);
    if (lift > p) p = lift;
    off += al(sizeof(float) * kPartialCTAs * p);
  }
  w.total = off;
  return w;
}

struct SavesMap {
  size_t act, xhat;
  size_t x(int l) const { return (size_t)l * (2 * act + xhat); }
  size_t pre(int l) const { return x(l) + act; }
  size_t xh(int l) const { return x(l) + 2 * act; }
  size_t vlast(int L) const { return x(L); }
  size_t total(int L) const { return x(L) + act; }
};

SavesMap saves_map(const fno_net_desc *d, const Geom &g) {
  SavesMap m;
  m.act = al(elsize(d->dtype) * (size_t)(g.B * d->width * g.N));
  m.xhat = al(sizeof(float2) * (size_t)(g.B * d->width * g.K));
  return m;
}

}  // namespace

namespace fno {

void set_last_error(const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

void launch_begin(const Launch &L) {
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (g_prof_used == g_prof.size()) {
    ProfRec r{};
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) {
      cudaGetLastError();
      return;
    }
    g_prof.push_back(r);
  }
  cudaEventRecord(g_prof[g_prof_used].start, L.stream);
}

void launch_end(const Launch &L, const char *tag) {
  ++*L.count;
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (g_prof_used >= g_prof.size()) return;
  cudaEventRecord(g_prof[g_prof_used].stop, L.stream);
  g_prof[g_prof_used].tag = tag;
  ++g_prof_used;
}

}  // namespace fno

// ===========================================================================
// public entry points
// ===========================================================================

extern "C" {

const char *fno_last_error(void) { return g_err; }

const char *fno_version(void) { return "fno-b200 0.1 (sm_100a)"; }

int fno_last_launch_count(void) { return g_launches; }

int fno_set_tensor_cores(int enable) {
  const int prev = g_use_tc;
  g_use_tc = (enable >= 2 && enable <= 4) ? enable : enable ? 1 : 0;
  return prev;
}

int fno_device_error(int clear) {
  int *p = device_error_word();
  if (!p) return fail(FNO_ERR_CUDA, "no CUDA device");
  int v = 0;
  cudaError_t e = cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (clear && v) {
    const int zero = 0;
    e = cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  }
  if (v) return fail(FNO_ERR_TIMEOUT, "a bounded device-side wait expired (results invalid)");
  g_err[0] = 0;
  return FNO_OK;
}

int fno_set_wait_limit(int spins) {
  if (spins < 0) return fail(FNO_ERR_INVALID_ARG, "wait limit %d < 0", spins);
  int *p = device_error_word();
  if (!p) return fail(FNO_ERR_CUDA, "no CUDA device");
  int prev = 0;
  cudaError_t e = cudaMemcpy(&prev, p + 1, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the wait limit");
  e = cudaMemcpy(p + 1, &spins, sizeof(int), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "setting the wait limit");
  g_err[0] = 0;
  return prev;
}

int fno_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (on) g_prof_used = 0;
  g_prof_on = on != 0;
  return FNO_OK;
}

int fno_profile_read(fno_kernel_stat *out, int max) {
  if (!out || max < 1) return fail(FNO_ERR_INVALID_ARG, "output array is NULL or empty");
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int n = 0;
  for (size_t i = 0; i < g_prof_used; ++i) {
    const ProfRec &r = g_prof[i];
    cudaError_t e = cudaEventSynchronize(r.stop);
    if (e != cudaSuccess) return cuda_fail(e, "profile read");
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, r.start, r.stop);
    if (e != cudaSuccess) return cuda_fail(e, "profile read");
    int j = 0;
    while (j < n && strcmp(out[j].name, r.tag) != 0) ++j;
    if (j == n) {
      if (n == max) continue;
      memset(&out[n], 0, sizeof(out[n]));
      snprintf(out[n].name, sizeof(out[n].name), "%s", r.tag);
      ++n;
    }
    out[j].launches += 1;
    out[j].total_ms += ms;
  }
  g_err[0] = 0;
  return n;
}

size_t fno_workspace_size(const fno_block_desc *desc, int op) {
  Geom g;
  if (check_block(desc, &g)) return 0;
  if (op < FNO_OP_SPECTRAL_FWD || op > FNO_OP_BLOCK_BWD_CP || op == FNO_OP_NET_FWD ||
      op == FNO_OP_NET_BWD) {
    fail(FNO_ERR_INVALID_ARG, "op %d is not a block op", op);
    return 0;
  }
  g_err[0] = 0;
  return block_ws(g, desc->cin, desc->cout, op).total;
}

size_t fno_net_workspace_size(const fno_net_desc *desc, int op) {
  Geom g;
  if (check_net(desc, &g)) return 0;
  if (op != FNO_OP_NET_FWD && op != FNO_OP_NET_BWD) {
    fail(FNO_ERR_INVALID_ARG, "op %d is not a network op", op);
    return 0;
  }
  g_err[0] = 0;
  return net_ws(desc, g, op).total;
}

size_t fno_net_saves_size(const fno_net_desc *desc) {
  Geom g;
  if (check_net(desc, &g)) return 0;
  g_err[0] = 0;
  return saves_map(desc, g).total(desc->n_layers);
}

int fno_spectral_conv_fwd(const fno_block_desc *desc, const void *x, const void *R, void *y,
                          float *xhat_save, void *ws, size_t ws_bytes, fno_stream_t stream) {
  Geom g;
  int rc = check_block(desc, &g);
  if (rc) return rc;
  if ((rc = check_smem(g, desc->cin, desc->cout, FNO_OP_SPECTRAL_FWD))) return rc;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(R, "R");
  REQUIRE_PTR(y, "y");
  OPTIONAL_PTR(xhat_save, "xhat_save");
  const size_t need = block_ws(g, desc->cin, desc->cout, FNO_OP_SPECTRAL_FWD).total;
  if (ws_bytes < need) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  rc = run_forward(L, g, desc->dtype, desc->flags, desc->cin, desc->cout, x, R, nullptr, nullptr,
                   y, nullptr, xhat_save, (unsigned char *)ws, EPI_SPEC);
  if (!rc) g_err[0] = 0;
  return rc;
}

int fno_spectral_conv_bwd(const fno_block_desc *desc, const void *x, const float *xhat_save,
                          const void *R, const void *dy, void *dx, float *dR, void *ws,
                          size_t ws_bytes, fno_stream_t stream) {
  Geom g;
  int rc = check_block(desc, &g);
  if (rc) return rc;
  if ((rc = check_smem(g, desc->cin, desc->cout, FNO_OP_SPECTRAL_BWD))) return rc;
  REQUIRE_PTR(x, "x");
  OPTIONAL_PTR(xhat_save, "xhat_save");
  REQUIRE_PTR(R, "R");
  REQUIRE_PTR(dy, "dy");
  REQUIRE_PTR(dx, "dx");
  REQUIRE_PTR(dR, "dR");
  const size_t need = block_ws(g, desc->cin, desc->cout, FNO_OP_SPECTRAL_BWD).total;
  if (ws_bytes < need) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  rc = run_backward(L, g, desc->dtype, desc->flags, desc->cin, desc->cout, x, xhat_save, R,
                    nullptr, nullptr, dy, dx, dR, nullptr, nullptr, (unsigned char *)ws, false);
  if (!rc) g_err[0] = 0;
  return rc;
}

int fno_block_fwd(const fno_block_desc *desc, const void *x, const void *R, const void *W,
                  const void *b, void *y, void *pre_save, float *xhat_save, void *ws,
                  size_t ws_bytes, fno_stream_t stream) {
  Geom g;
  int rc = check_block(desc, &g);
  if (rc) return rc;
  if ((rc = check_smem(g, desc->cin, desc->cout, FNO_OP_BLOCK_FWD))) return rc;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(R, "R");
  REQUIRE_PTR(W, "W");
  REQUIRE_PTR(b, "b");
  REQUIRE_PTR(y, "y");
  OPTIONAL_PTR(pre_save, "pre_save");
  OPTIONAL_PTR(xhat_save, "xhat_save");
  const size_t need = block_ws(g, desc->cin, desc->cout, FNO_OP_BLOCK_FWD).total;
  if (ws_bytes < need) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  rc = run_forward(L, g, desc->dtype, desc->flags, desc->cin, desc->cout, x, R, W, b, y, pre_save,
                   xhat_save, (unsigned char *)ws, EPI_BLOCK_FWD);
  if (!rc) g_err[0] = 0;
  return rc;
}

static int check_cp(const fno_block_desc *desc, int rank, const void *lam,
                    const void *A, const void *B, const void *C) {
  if (rank < 1) return fail(FNO_ERR_INVALID_ARG, "rank %d < 1", rank);
  if (rank > kMaxCpRank)
    return fail(FNO_ERR_UNSUPPORTED, "rank %d exceeds %d", rank, kMaxCpRank);
  REQUIRE_PTR(lam, "lam");
  REQUIRE_PTR(A, "A");
  REQUIRE_PTR(B, "B");
  REQUIRE_PTR(C, "C");
  const size_t smem = sizeof(float2) * (size_t)(desc->cin + desc->cout) * kMaxCpRank;
  if (smem > kSmemLimit) return fail(FNO_ERR_UNSUPPORTED, "factor staging needs %zu B", smem);
  return FNO_OK;
}

int fno_spectral_conv_fwd_cp(const fno_block_desc *desc, int rank, const void *x, const void *lam,
                             const void *A, const void *B, const void *C, void *y,
                             float *xhat_save, void *ws, size_t ws_bytes, fno_stream_t stream) {
  Geom g;
  int rc = check_block(desc, &g);
  if (rc) return rc;
  if ((rc = check_smem(g, desc->cin, desc->cout, FNO_OP_SPECTRAL_FWD))) return rc;
  if ((rc = check_cp(desc, rank, lam, A, B, C))) return rc;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(y, "y");
  OPTIONAL_PTR(xhat_save, "xhat_save");
  const size_t need = block_ws(g, desc->cin, desc->cout, FNO_OP_SPECTRAL_FWD).total;
  if (ws_bytes < need) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  const CpFactors f{lam, A, B, C};
  rc = run_forward(L, g, desc->dtype, desc->flags, desc->cin, desc->cout, x, nullptr, nullptr,
                   nullptr, y, nullptr, xhat_save, (unsigned char *)ws, EPI_SPEC, &f, rank);
  if (!rc) g_err[0] = 0;
  return rc;
}

int fno_block_fwd_cp(const fno_block_desc *desc, int rank, const void *x, const void *lam,
                     const void *A, const void *B, const void *C, const void *W, const void *b,
                     void *y, void *pre_save, float *xhat_save, void *ws, size_t ws_bytes,
                     fno_stream_t stream) {
  Geom g;
  int rc = check_block(desc, &g);
  if (rc) return rc;
  if ((rc = check_smem(g, desc->cin, desc->cout, FNO_OP_BLOCK_FWD))) return rc;
  if ((rc = check_cp(desc, rank, lam, A, B, C))) return rc;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(W, "W");
  REQUIRE_PTR(b, "b");
  REQUIRE_PTR(y, "y");
  OPTIONAL_PTR(pre_save, "pre_save");
  OPTIONAL_PTR(xhat_save, "xhat_save");
  const size_t need = block_ws(g, desc->cin, desc->cout, FNO_OP_BLOCK_FWD).total;
  if (ws_bytes < need) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  const CpFactors f{lam, A, B, C};
  rc = run_forward(L, g, desc->dtype, desc->flags, desc->cin, desc->cout, x, nullptr, W, b, y,
                   pre_save, xhat_save, (unsigned char *)ws, EPI_BLOCK_FWD, &f, rank);
  if (!rc) g_err[0] = 0;
  return rc;
}

static int bwd_cp(const fno_block_desc *desc, int rank, const void *x, const void *lam,
                  const void *A, const void *B, const void *C, const void *W, const void *pre_save,
                  const float *xhat_save, const void *dy, void *dx, float *dlam, float *dA,
                  float *dB, float *dC, float *dW, float *db, void *ws, size_t ws_bytes,
                  fno_stream_t stream, bool block) {
  Geom g;
  int rc = check_block(desc, &g);
  if (rc) return rc;
  const int op = block ? FNO_OP_BLOCK_BWD_CP : FNO_OP_SPECTRAL_BWD_CP;
  if ((rc = check_smem(g, desc->cin, desc->cout, block ? FNO_OP_BLOCK_BWD : FNO_OP_SPECTRAL_BWD)))
    return rc;
  if ((rc = check_cp(desc, rank, lam, A, B, C))) return rc;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(dy, "dy");
  REQUIRE_PTR(dx, "dx");
  REQUIRE_PTR(dlam, "dlam");
  REQUIRE_PTR(dA, "dA");
  REQUIRE_PTR(dB, "dB");
  REQUIRE_PTR(dC, "dC");
  OPTIONAL_PTR(xhat_save, "xhat_save");
  if (block) {
    REQUIRE_PTR(W, "W");
    if (!(desc->flags & FNO_NO_ACT)) REQUIRE_PTR(pre_save, "pre_save");
    REQUIRE_PTR(dW, "dW");
    REQUIRE_PTR(db, "db");
  }
  const BlockWs w = block_ws(g, desc->cin, desc->cout, op);
  if (ws_bytes < w.total) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, w.total);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  unsigned char *wsb = (unsigned char *)ws;
  const CpFactors f{lam, A, B, C};
  void *R = wsb + w.rcp;
  float *dR = reinterpret_cast<float *>(wsb + w.drcp);
  FNO_TRY(launch_cp_rebuild(L, g, desc->dtype, desc->cin, desc->cout, rank, f, R),
          "factorised weight rebuild");
  rc = run_backward(L, g, desc->dtype, desc->flags, desc->cin, desc->cout, x, xhat_save, R, W,
                    pre_save, dy, dx, dR, dW, db, wsb, block, op);
  if (rc) return rc;
  FNO_TRY(launch_cp_grads(L, g, desc->dtype, desc->cin, desc->cout, rank, f, dR,
                          reinterpret_cast<float *>(wsb + w.cps), dlam, dA, dB, dC),
          "factor gradients");
  g_err[0] = 0;
  return FNO_OK;
}

int fno_spectral_conv_bwd_cp(const fno_block_desc *desc, int rank, const void *x,
                             const void *lam, const void *A, const void *B, const void *C,
                             const float *xhat_save, const void *dy, void *dx, float *dlam,
                             float *dA, float *dB, float *dC, void *ws, size_t ws_bytes,
                             fno_stream_t stream) {
  return bwd_cp(desc, rank, x, lam, A, B, C, nullptr, nullptr, xhat_save, dy, dx, dlam, dA, dB,
                dC, nullptr, nullptr, ws, ws_bytes, stream, false);
}

int fno_block_bwd_cp(const fno_block_desc *desc, int rank, const void *x, const void *lam,
                     const void *A, const void *B, const void *C, const void *W,
                     const void *pre_save, const float *xhat_save, const void *dy, void *dx,
                     float *dlam, float *dA, float *dB, float *dC, float *dW, float *db, void *ws,
                     size_t ws_bytes, fno_stream_t stream) {
  return bwd_cp(desc, rank, x, lam, A, B, C, W, pre_save, xhat_save, dy, dx, dlam, dA, dB, dC, dW,
                db, ws, ws_bytes, stream, true);
}

int fno_block_bwd(const fno_block_desc *desc, const void *x, const void *R, const void *W,
                  const void *pre_save, const float *xhat_save, const void *dy, void *dx,
                  float *dR, float *dW, float *db, void *ws, size_t ws_bytes,
                  fno_stream_t stream) {
  Geom g;
  int rc = check_block(desc, &g);
  if (rc) return rc;
  if ((rc = check_smem(g, desc->cin, desc->cout, FNO_OP_BLOCK_BWD))) return rc;
  REQUIRE_PTR(x, "x");
  REQUIRE_PTR(R, "R");
  REQUIRE_PTR(W, "W");
  if (!(desc->flags & FNO_NO_ACT)) REQUIRE_PTR(pre_save, "pre_save");
  OPTIONAL_PTR(xhat_save, "xhat_save");
  REQUIRE_PTR(dy, "dy");
  REQUIRE_PTR(dx, "dx");
  REQUIRE_PTR(dR, "dR");
  REQUIRE_PTR(dW, "dW");
  REQUIRE_PTR(db, "db");
  const size_t need = block_ws(g, desc->cin, desc->cout, FNO_OP_BLOCK_BWD).total;
  if (ws_bytes < need) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, need);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  rc = run_backward(L, g, desc->dtype, desc->flags, desc->cin, desc->cout, x, xhat_save, R, W,
                    pre_save, dy, dx, dR, dW, db, (unsigned char *)ws, true);
  if (!rc) g_err[0] = 0;
  return rc;
}

int fno_forward(const fno_net_desc *desc, const void *a, const fno_params *params, void *u,
                void *saves, void *ws, size_t ws_bytes, fno_stream_t stream) {
  Geom g;
  int rc = check_net(desc, &g);
  if (rc) return rc;
  REQUIRE_PTR(a, "a");
  if (!params) return fail(FNO_ERR_INVALID_ARG, "params is NULL");
  REQUIRE_PTR(params->P, "P");
  REQUIRE_PTR(params->p, "p");
  REQUIRE_PTR(params->Q1, "Q1");
  REQUIRE_PTR(params->q1, "q1");
  REQUIRE_PTR(params->Q2, "Q2");
  REQUIRE_PTR(params->q2, "q2");
  for (int l = 0; l < desc->n_layers; ++l) {
    REQUIRE_PTR(params->R[l], "R[l]");
    REQUIRE_PTR(params->W[l], "W[l]");
    REQUIRE_PTR(params->b[l], "b[l]");
  }
  REQUIRE_PTR(u, "u");
  OPTIONAL_PTR(saves, "saves");
  const NetWs w = net_ws(desc, g, FNO_OP_NET_FWD);
  if (ws_bytes < w.total) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, w.total);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  unsigned char *wsb = (unsigned char *)ws;
  unsigned char *sv = (unsigned char *)saves;
  const SavesMap sm = saves_map(desc, g);
  const int nl = desc->n_layers;
  auto act_buf = [&](int l) -> void * {  // input of block l (l == nl: projection input)
    if (sv) return sv + (l < nl ? sm.x(l) : sm.vlast(nl));
    return wsb + ((l & 1) ? w.act1 : w.act0);
  };
  FNO_TRY(launch_lift(L, g, desc->dtype, desc->in_channels, desc->width, a, params->P, params->p,
                      act_buf(0)),
          "lift");
  for (int l = 0; l < nl; ++l) {
    rc = run_forward(L, g, desc->dtype, desc->flags, desc->width, desc->width, act_buf(l),
                     params->R[l], params->W[l], params->b[l], act_buf(l + 1),
                     sv ? sv + sm.pre(l) : nullptr,
                     sv ? reinterpret_cast<float *>(sv + sm.xh(l)) : nullptr, wsb + w.block,
                     EPI_BLOCK_FWD);
    if (rc) return rc;
  }
  FNO_TRY(launch_proj_fwd(L, g, desc->dtype, desc->width, desc->hidden, desc->out_channels,
                          act_buf(nl), params->Q1, params->q1, params->Q2, params->q2, u),
          "projection");
  g_err[0] = 0;
  return FNO_OK;
}

int fno_backward(const fno_net_desc *desc, const void *a, const fno_params *params,
                 const void *saves, const void *du, fno_grads *grads, void *ws, size_t ws_bytes,
                 fno_stream_t stream) {
  return fno_backward_ready(desc, a, params, saves, du, grads, ws, ws_bytes, stream, nullptr, 0);
}

int fno_backward_ready(const fno_net_desc *desc, const void *a, const fno_params *params,
                       const void *saves, const void *du, fno_grads *grads, void *ws,
                       size_t ws_bytes, fno_stream_t stream, fno_event_t *ready, int n_ready) {
  Geom g;
  int rc = check_net(desc, &g);
  if (rc) return rc;
  if (ready || n_ready) {
    if (!ready || n_ready != desc->n_layers + 2)
      return fail(FNO_ERR_INVALID_ARG, "ready needs n_layers + 2 = %d events (got %d%s)",
                  desc->n_layers + 2, n_ready, ready ? "" : ", array NULL");
    for (int j = 0; j < n_ready; ++j)
      if (!ready[j]) return fail(FNO_ERR_INVALID_ARG, "ready[%d] is NULL", j);
  }
  REQUIRE_PTR(a, "a");
  if (!params) return fail(FNO_ERR_INVALID_ARG, "params is NULL");
  if (!grads) return fail(FNO_ERR_INVALID_ARG, "grads is NULL");
  REQUIRE_PTR(saves, "saves");
  REQUIRE_PTR(du, "du");
  REQUIRE_PTR(params->Q1, "Q1");
  REQUIRE_PTR(params->q1, "q1");
  REQUIRE_PTR(params->Q2, "Q2");
  REQUIRE_PTR(grads->P, "dP");
  REQUIRE_PTR(grads->p, "dp");
  REQUIRE_PTR(grads->Q1, "dQ1");
  REQUIRE_PTR(grads->q1, "dq1");
  REQUIRE_PTR(grads->Q2, "dQ2");
  REQUIRE_PTR(grads->q2, "dq2");
  for (int l = 0; l < desc->n_layers; ++l) {
    REQUIRE_PTR(params->R[l], "R[l]");
    REQUIRE_PTR(params->W[l], "W[l]");
    REQUIRE_PTR(grads->R[l], "dR[l]");
    REQUIRE_PTR(grads->W[l], "dW[l]");
    REQUIRE_PTR(grads->b[l], "db[l]");
  }
  const NetWs w = net_ws(desc, g, FNO_OP_NET_BWD);
  if (ws_bytes < w.total) return fail(FNO_ERR_WORKSPACE, "workspace %zu B < %zu B", ws_bytes, w.total);
  REQUIRE_PTR(ws, "ws");
  Launch L = make_launch(stream);
  unsigned char *wsb = (unsigned char *)ws;
  const unsigned char *sv = (const unsigned char *)saves;
  const SavesMap sm = saves_map(desc, g);
  const int nl = desc->n_layers;
  const int width = desc->width, hidden = desc->hidden, outc = desc->out_channels;
  float *partial = reinterpret_cast<float *>(wsb + w.partial);
  void *dv[2] = {wsb + w.act0, wsb + w.act1};

  int np = proj_bwd_grid(g, L.num_sms);
  if ((L.tc == 1 || L.tc == 3 || L.tc == 4) &&
      proj_bwd_pipe_supported(g, desc->dtype, width, hidden, outc, sv + sm.vlast(nl), du,
                              dv[nl & 1])) {
    FNO_TRY(launch_proj_bwd_pipe(L, g, desc->dtype, width, hidden, outc, sv + sm.vlast(nl), du,
                                 params->Q1, params->q1, params->Q2, dv[nl & 1], partial, &np),
            "projection backward");
  } else {
    FNO_TRY(launch_proj_bwd(L, g, desc->dtype, width, hidden, outc, sv + sm.vlast(nl), du,
                            params->Q1, params->q1, params->Q2, dv[nl & 1], partial),
            "projection backward");
  }
  const long long pstride = (long long)proj_bwd_partial_floats(width, hidden, outc);
  FNO_TRY(launch_reduce_rows(L, partial, np, pstride, 0, hidden, width, grads->Q1, grads->q1),
          "dQ1 reduction");
  FNO_TRY(launch_reduce_rows(L, partial, np, pstride, (long long)hidden * (width + 1), outc,
                             hidden, grads->Q2, grads->q2),
          "dQ2 reduction");
  if (ready) FNO_TRY(cudaEventRecord(ready[0], L.stream), "recording ready[0]");
  for (int l = nl - 1; l >= 0; --l) {
    rc = run_backward(L, g, desc->dtype, desc->flags, width, width, sv + sm.x(l),
                      reinterpret_cast<const float *>(sv + sm.xh(l)), params->R[l], params->W[l],
                      sv + sm.pre(l), dv[(l + 1) & 1], dv[l & 1], grads->R[l], grads->W[l],
                      grads->b[l], wsb + w.block, true);
    if (rc) return rc;
    if (ready) FNO_TRY(cudaEventRecord(ready[nl - l], L.stream), "recording a layer's ready event");
  }
  FNO_TRY(launch_lift_bwd(L, g, desc->dtype, desc->in_channels, width, a, dv[0], partial),
          "lift backward");
  const int nl2 = lift_bwd_grid(g, L.num_sms);
  FNO_TRY(launch_reduce_rows(L, partial, nl2, (long long)width * (desc->in_channels + 1), 0, width,
                             desc->in_channels, grads->P, grads->p),
          "dP reduction");
  if (ready) FNO_TRY(cudaEventRecord(ready[nl + 1], L.stream), "recording ready[L + 1]");
  g_err[0] = 0;
  return FNO_OK;
}

int fno_mse(int64_t n, int dtype, const void *u, const void *target, float *loss, void *du,
            fno_stream_t stream) {
  if (n < 1) return fail(FNO_ERR_INVALID_ARG, "n %lld < 1", (long long)n);
  if (dtype < FNO_F32 || dtype > FNO_BF16) return fail(FNO_ERR_INVALID_ARG, "dtype %d unknown", dtype);
  REQUIRE_PTR(u, "u");
  REQUIRE_PTR(target, "target");
  if (!loss) return fail(FNO_ERR_INVALID_ARG, "loss is NULL");
  OPTIONAL_PTR(du, "du");
  Launch L = make_launch(stream);
  FNO_TRY(launch_mse(L, n, dtype, u, target, loss, du), "mse");
  g_err[0] = 0;
  return FNO_OK;
}

int fno_adam_step(int64_t n, float *theta, float *m, float *v, const float *grad,
                  void *param_out, int out_dtype, int step, float lr, float beta1, float beta2,
                  float eps, float weight_decay, float grad_scale, fno_stream_t stream) {
  if (n < 1) return fail(FNO_ERR_INVALID_ARG, "n %lld < 1", (long long)n);
  REQUIRE_PTR(theta, "theta");
  OPTIONAL_PTR(param_out, "param_out");
  if (param_out && (out_dtype < FNO_F32 || out_dtype > FNO_BF16))
    return fail(FNO_ERR_INVALID_ARG, "out_dtype %d unknown", out_dtype);
  AdamCoef c{};
  if (grad) {
    REQUIRE_PTR(grad, "grad");
    REQUIRE_PTR(m, "m");
    REQUIRE_PTR(v, "v");
    if (step < 1) return fail(FNO_ERR_INVALID_ARG, "step %d < 1", step);
    if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
      return fail(FNO_ERR_INVALID_ARG, "betas (%g, %g) not in [0, 1)", beta1, beta2);
    if (!(eps > 0.f) || !isfinite(eps)) return fail(FNO_ERR_INVALID_ARG, "eps %g <= 0", eps);
    if (!(lr >= 0.f) || !isfinite(lr)) return fail(FNO_ERR_INVALID_ARG, "lr %g < 0", lr);
    if (!(weight_decay >= 0.f) || !isfinite(weight_decay))
      return fail(FNO_ERR_INVALID_ARG, "weight_decay %g < 0", weight_decay);
    if (!isfinite(grad_scale)) return fail(FNO_ERR_INVALID_ARG, "grad_scale is not finite");
    c.lr = lr;
    c.beta1 = beta1;
    c.beta2 = beta2;
    c.one_minus_beta1 = (float)(1.0 - (double)beta1);
    c.one_minus_beta2 = (float)(1.0 - (double)beta2);
    c.inv_bc1 = (float)(1.0 / (1.0 - pow((double)beta1, (double)step)));
    c.inv_bc2 = (float)(1.0 / (1.0 - pow((double)beta2, (double)step)));
    c.eps = eps;
    c.lr_wd = (float)((double)lr * (double)weight_decay);
    c.grad_scale = grad_scale;
  } else if (!param_out) {
    return fail(FNO_ERR_INVALID_ARG, "neither grad nor param_out given: nothing to do");
  }
  Launch L = make_launch(stream);
  FNO_TRY(launch_adam(L, n, theta, grad ? m : nullptr, grad ? v : nullptr, grad, param_out,
                      out_dtype, c),
          "adam");
  g_err[0] = 0;
  return FNO_OK;
}

}  // extern "C"
