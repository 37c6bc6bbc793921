// Internal kernel interface of the FNO library: geometry, argument blocks and
// launchers.  Nothing here is part of the public C ABI (include/fno.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace fno {

constexpr int kMaxWidth = 64;   // channels held in registers per grid point
constexpr int kMaxAxis = 4096;  // longest axis whose twiddle table fits shared memory

// Grid geometry of one block, flattened to at most three axes:
//   outer axis (d == 3: axis 0), slab axis (d >= 2: axis d-2), last axis.
// Missing axes have length 1 and a single kept mode.
struct Geom {
  int d;
  long long B;
  int O, mO, QO;    // outer axis length, modes, kept count (2 mO or 1)
  int S, mS, QS;    // slab axis
  int NL, mL;       // last (real-FFT) axis
  long long N;      // points per channel = O * S * NL
  long long K;      // kept modes = QO * QS * mL
  float inv_n;      // 1 / N
};

enum LoadMode { LOAD_PLAIN = 0, LOAD_TANH = 1, LOAD_DZ = 2 };
enum EpiMode { EPI_SPEC = 0, EPI_BLOCK_FWD = 1, EPI_SPEC_BWD = 2, EPI_BLOCK_BWD = 3 };

// dtype codes match include/fno.h
enum { DT_F32 = 0, DT_F16 = 1, DT_BF16 = 2 };

struct Launch {
  cudaStream_t stream;
  int *count;       // incremented per kernel launch
  int num_sms;
  int tc;           // 1: default (pruned-FFT transform, mixing and pruned slab-axis
                    //    inverse on CUDA cores where each is measured faster, tcgen05
                    //    mixing for bf16 weights at 64 outputs, tcgen05 TMA pipelines
                    //    for the epilogue and projection);
                    // 4: as 1 with the clustered FFT transform;
                    // 3: tcgen05 TMA pipelines throughout (dense DFT-matrix transform);
                    // 2: tcgen05 without the pipelines; 0: CUDA cores only
  int *err;         // device error word (bounded waits that expired)
};

// Set the thread-local message fno_last_error() returns.
void set_last_error(const char *fmt, ...);

// Bracket every kernel launch: launch_begin records a CUDA event on the launch
// stream when per-kernel timing is on (fno_profile_enable); launch_end records
// the closing event under `tag` and counts the launch.
void launch_begin(const Launch &L);
void launch_end(const Launch &L, const char *tag);

// ---- forward truncated transform (S0-S2) ----------------------------------
// in0 (and in1 for LOAD_DZ) are [B][C][N]; out xhat [B][C][K] float2.
// zpart scratch: fwd_zpart_floats() floats.
int fwd_bands(const Geom &g, long long planes, int num_sms);
size_t fwd_zpart_bytes(const Geom &g, long long C);
cudaError_t launch_fwd_transform(const Launch &L, const Geom &g, int dtype, int load_mode,
                                 long long C, const void *in0, const void *in1, float2 *zpart,
                                 float2 *xhat);

// ---- tensor-core variants (transform_tc.cu, epilogue_tc.cu) ----------------
bool s1_tc_supported(const Geom &g, int dtype);
int s1_tc_bands(const Geom &g);
cudaError_t launch_s1_tc(const Launch &L, const Geom &g, int dtype, int load_mode, long long C,
                         const void *in0, const void *in1, float2 *zpart, int *err);

// warp-specialised TMA pipeline for the forward transform (LOAD_PLAIN /
// LOAD_TANH): writes the same per-band partial sums as launch_s1_tc
bool fwd_pipe_supported(const Geom &g, int dtype, int load_mode, const void *in0);
cudaError_t launch_fwd_pipe(const Launch &L, const Geom &g, int dtype, int load_mode,
                            long long C, const void *in0, float2 *zpart);

// pruned radix-16 FFT transform on the CUDA cores (transform_fft.cu): one
// thread-block cluster per plane writes out[plane][QS][mL] (for 2D grids that
// is xhat itself; for 3D the outer axis is still to be contracted)
bool fwd_fft_supported(const Geom &g, const void *in0, const void *in1, int load_mode);
cudaError_t launch_fwd_fft(const Launch &L, const Geom &g, int dtype, int load_mode, long long C,
                           const void *in0, const void *in1, float2 *out);

// the same transform with whole planes per persistent CTA (transform_plane.cu):
// rows streamed by bulk async copies, slab axis as a pruned FFT on chip;
// writes out[plane][QS][mL] like launch_fwd_fft
bool fwd_plane_supported(const Geom &g, int dtype, const void *in0, const void *in1,
                         int load_mode);
cudaError_t launch_fwd_plane(const Launch &L, const Geom &g, int dtype, int load_mode, long long C,
                             const void *in0, const void *in1, float2 *out);

// 2D spectral middle (spec_mid.cu): mixing into yhat (launch_mix_fwd), then
// the slab-axis inverse as a pruned FFT into
// U[b][o][S][mL] = sum_q yhat[b,o,q,k] exp(+2 pi i kq n / S); two launches.
// img (optional): write the epilogue's B images (epi_img_supported and
// spec_mid_img_supported) instead of U, with bias (may be NULL) folded in
bool spec_mid_supported(const Geom &g, int Ci, int Co);
bool spec_mid_img_supported(const Geom &g, int Co);
cudaError_t launch_spec_mid(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                            const float2 *xhat, const void *R, float2 *yhat, float2 *U,
                            unsigned char *img, const void *bias);
// the pruned slab-axis inverse alone (the backward's dxhat), same output as
// launch_inv_slab: U[b][c][S][mL]
bool inv_slab_fft_supported(const Geom &g);
cudaError_t launch_inv_slab_fft(const Launch &L, const Geom &g, long long C, const float2 *Z,
                                float2 *U);

// CP-factorised weights (mix_cp.cu): R[i,o,k] = sum_r lam[r] A[i,r] B[o,r] C[k,r],
// factors complex (re, im) in the storage dtype: lam [rank], A [Ci][rank],
// B [Co][rank], C [K][rank]; yhat as launch_mix_fwd writes it
constexpr int kMaxCpRank = 32;
struct CpFactors {
  const void *lam, *A, *B, *C;
};
cudaError_t launch_mix_cp(const Launch &L, const Geom &g, int dtype, int Ci, int Co, int rank,
                          const float2 *xhat, const CpFactors &f, float2 *yhat);
// backward through the factors: the dense weight rebuilt in the storage dtype
// (R [Ci][Co][K][2]) for the dense backward, then from its gradient dR
// (float32 [Ci][Co][K][2]) the factor gradients (float32, (re, im)):
// dlam [rank], dA [Ci][rank], dB [Co][rank], dC [K][rank]; scratch: Ci rank
// complex floats
cudaError_t launch_cp_rebuild(const Launch &L, const Geom &g, int dtype, int Ci, int Co, int rank,
                              const CpFactors &f, void *R);
cudaError_t launch_cp_grads(const Launch &L, const Geom &g, int dtype, int Ci, int Co, int rank,
                            const CpFactors &f, const float *dR, float *scratch, float *dlam,
                            float *dA, float *dB, float *dC);

// ---- mixing (S3) -----------------------------------------------------------
// yhat[b,o,k] = (c_k / N) sum_i xhat[b,i,k] R[i,o,k]
// tcgen05 mixing (mix_tc.cu): bfloat16 weights, 64 output channels (Co for
// the forward, Ci for the adjoint dxhat), batch <= 64, K a multiple of 4
bool mix_tc_supported(const Geom &g, int dtype, bool adj, int Ci, int Co, const void *X,
                      const void *R, const void *Y);
cudaError_t launch_mix_tc(const Launch &L, const Geom &g, bool adj, int Ci, int Co,
                          const float2 *X, const void *R, float2 *Y);
cudaError_t launch_mix_fwd(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                           const float2 *xhat, const void *R, float2 *yhat);
// dR[i,o,k] = sum_b conj(xhat[b,i,k]) (c_k/N) D[b,o,k]
cudaError_t launch_mix_bwd_dr(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                              const float2 *xhat, const float2 *D, float *dR);
// tcgen05 dR (mix_tc.cu): 16-bit storage, 64 input channels, batch <= 64
bool mix_tc_dr_supported(const Geom &g, int dtype, int Ci, int Co, const void *X, const void *D,
                         const void *dR);
cudaError_t launch_mix_tc_dr(const Launch &L, const Geom &g, int Co, const float2 *X,
                             const float2 *D, float *dR);
// dxhat[b,i,k] = sum_o (c_k/N) D[b,o,k] conj(R[i,o,k])
cudaError_t launch_mix_bwd_dx(const Launch &L, const Geom &g, int dtype, int Ci, int Co,
                              const float2 *D, const void *R, float2 *dxhat);

// ---- inverse of the outer axis (d == 3) -----------------------------------
size_t inv_expand_bytes(const Geom &g, long long C);
cudaError_t launch_inv_expand(const Launch &L, const Geom &g, long long C, const float2 *V,
                              float2 *Z);

// ---- inverse of slab + last axis with fused epilogue (S4, S6 epilogue) ----
struct EpiArgs {
  const float2 *Z;  // [B][Cs][O][QS][mL]
  const void *x;    // [B][Ci][N]
  const void *W;    // [Co][Ci]
  const void *bias; // [Co]
  const void *dy;   // [B][Co][N]
  const void *pre;  // [B][Co][N]
  void *out;        // y (fwd modes, [B][Co][N]) or dx (bwd modes, [B][Ci][N])
  void *pre_out;    // optional [B][Co][N]
  float *partial;   // bwd: per-CTA partial sums of dW/db, [grid][Co][Ci+1]
  const float2 *U;  // optional: the spectrum already inverted along the slab axis,
                    // [B][Cs][O][S][mL] (launch_inv_slab); NULL: computed per tile
  const unsigned char *img;  // optional (pipelined forward epilogue): per grid row the
                             // spectral half of the B operand, prebuilt (launch_spec_mid)
  int Ci, Co;
  int act, tanh_pre;
};
int epi_grid(const Geom &g, int mode, int num_sms);
// tensor-core epilogue: U = spectrum inverted along the slab axis,
// [B][Cs][O][S][mL] float2 (launch_inv_slab), then one GEMM per 128-point tile
bool epi_tc_supported(const Geom &g, int dtype, int mode, int Ci, int Co);
size_t inv_slab_bytes(const Geom &g, long long C);
cudaError_t launch_inv_slab(const Launch &L, const Geom &g, long long C, const float2 *Z,
                            float2 *U);
struct EpiArgs;
cudaError_t launch_epilogue_tc(const Launch &L, const Geom &g, int dtype, int mode,
                               const EpiArgs &a, const float2 *U);
// warp-specialised TMA pipeline for the forward epilogue modes (EPI_SPEC,
// EPI_BLOCK_FWD); same inputs as launch_epilogue_tc
bool epi_pipe_supported(const Geom &g, int dtype, int mode, int Ci, int Co, const void *x,
                        const void *U);
cudaError_t launch_epi_pipe(const Launch &L, const Geom &g, int dtype, int mode,
                            const EpiArgs &a, const float2 *U);
// the prebuilt-image form (a.img): 2D, last axis >= 128, Co % 16 == 0, 2 mL % 16 == 0.
// One image per (sample, grid row): the K-major no-swizzle core-matrix layout of
// the B operand rows o (float32: tf32 high parts in rows [0, Co), low parts in
// [Co, 2 Co)) by columns 2k (re), 2k + 1 (im), bias folded into column 0
bool epi_img_supported(const Geom &g, int dtype, int mode, int Ci, int Co);
size_t epi_img_row_bytes(int dtype, int Co, int mL);
// warp-specialised tcgen05 block backward (EPI_BLOCK_BWD), 16-bit storage, no
// tanh pre-activation, d >= 2, Ci and Co multiples of 16: dx, and per-CTA
// partials of dW / db in a.partial ([*nparts][Co][Ci + 1]); U = dxhat inverted
// along the slab axis ([B][Ci][O][S][mL] float2)
bool epi_bwd_pipe_supported(const Geom &g, int dtype, int Ci, int Co, int tanh_pre,
                            const void *x, const void *dy, const void *pre, int act,
                            const void *U);
cudaError_t launch_epi_bwd_pipe(const Launch &L, const Geom &g, int dtype, const EpiArgs &a,
                                const float2 *U, int *nparts);
size_t epi_partial_bytes(const Geom &g, int Ci, int Co, int num_sms);
cudaError_t launch_epilogue(const Launch &L, const Geom &g, int dtype, int mode,
                            const EpiArgs &a);

size_t epi_smem_bytes(const Geom &g, int mode, int Ci, int Co);

// Sum per-CTA partials: partial[p * stride + offset + r * (cols + 1) + c] over p
// into out_main[r * cols + c] (c < cols) and out_last[r] (c == cols); float32,
// overwritten.  Either output may be NULL.
cudaError_t launch_reduce_rows(const Launch &L, const float *partial, int nparts,
                               long long stride, long long offset, int rows, int cols,
                               float *out_main, float *out_last);

// CTAs of every kernel that writes per-CTA partial sums (fixed, so workspace
// sizes do not depend on the device).
constexpr int kPartialCTAs = 296;

// ---- lift / projection / loss (S5) ----------------------------------------
cudaError_t launch_lift(const Launch &L, const Geom &g, int dtype, int in_ch, int width,
                        const void *a, const void *P, const void *p, void *v);
cudaError_t launch_proj_fwd(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                            int out_ch, const void *v, const void *Q1, const void *q1,
                            const void *Q2, const void *q2, void *u);
bool proj_tc_supported(const Geom &g, int dtype, int width, int hidden, int out_ch);
// warp-specialised TMA pipeline for the projection
bool proj_pipe_supported(const Geom &g, int dtype, int width, int hidden, int out_ch,
                         const void *v);
cudaError_t launch_proj_pipe(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                             int out_ch, const void *v, const void *Q1, const void *q1,
                             const void *Q2, const void *q2, void *u);
cudaError_t launch_proj_fwd_tc(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                               int out_ch, const void *v, const void *Q1, const void *q1,
                               const void *Q2, const void *q2, void *u);
// tcgen05 projection backward, 16-bit storage, width % 16 == 0, hidden <= 128:
// dv, and per-CTA partials in the layout of launch_proj_bwd (*nparts of them)
bool proj_bwd_pipe_supported(const Geom &g, int dtype, int width, int hidden, int out_ch,
                             const void *v, const void *du, const void *dv);
cudaError_t launch_proj_bwd_pipe(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                                 int out_ch, const void *v, const void *du, const void *Q1,
                                 const void *q1, const void *Q2, void *dv, float *partial,
                                 int *nparts);
int proj_bwd_grid(const Geom &g, int num_sms);
size_t proj_bwd_partial_floats(int width, int hidden, int out_ch);
size_t proj_bwd_smem_bytes(int width, int hidden, int out_ch);
cudaError_t launch_proj_bwd(const Launch &L, const Geom &g, int dtype, int width, int hidden,
                            int out_ch, const void *v, const void *du, const void *Q1,
                            const void *q1, const void *Q2, void *dv, float *partial);
int lift_bwd_grid(const Geom &g, int num_sms);
cudaError_t launch_lift_bwd(const Launch &L, const Geom &g, int dtype, int in_ch, int width,
                            const void *a, const void *dv, float *partial);
cudaError_t launch_mse(const Launch &L, long long n, int dtype, const void *u, const void *t,
                       float *loss, void *du);

// Adam on float32 master weights fused with their storage-dtype copy
// (optim.cu).  g == nullptr: copy only; out == nullptr: update only.
struct AdamCoef {
  float lr, beta1, beta2, one_minus_beta1, one_minus_beta2;
  float inv_bc1, inv_bc2;   // 1 / (1 - beta^t)
  float eps, lr_wd, grad_scale;
};
cudaError_t launch_adam(const Launch &L, long long n, float *theta, float *m, float *v,
                        const float *g, void *out, int out_dtype, const AdamCoef &c);

}  // namespace fno
