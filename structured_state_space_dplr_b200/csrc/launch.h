// launch.h -- internal host-side launchers (one per kernel family).
#pragma once
#include <cuda_runtime.h>
#include <cstddef>

namespace s4 {

// remember a failing CUDA call for s4_last_cuda_error() (calling host thread)
void record_cuda_error(cudaError_t e);

// ---- spectral.cu: FFT convolution and inverse real FFT ----
// Cluster split used for the length-2L convolution transforms.
struct ConvGeom { int C; int lg; };
ConvGeom conv_geom(int L);
size_t conv_workspace_bytes(int H, int L);

// spectrum of K + D delta_0 (D may be null: no feed-through) into ws; with Ki
// (L > 8192 only) the spectrum of the complex signal K + i Ki instead
cudaError_t launch_kspec(const float *K, const float *D, int H, int L, void *ws, cudaStream_t st,
                         const float *Ki = nullptr);
// adjoint: the correlation with the same spectrum (conjugated), y[s] = sum_{t>=s} K[t-s] u[t] + D u[s]
cudaError_t launch_fftconv(const float *u, const void *ws, int Bt, int H, int L, float *y, cudaStream_t st,
                           bool adjoint = false);
// in place: K[H, L] holds the packed half spectrum on entry, the real kernel on exit
// ---- backward.cu ----
size_t corr_workspace_bytes(int H, int L);
cudaError_t launch_corr(const float *u, const float *dy, int Bt, int H, int L, float *dK, float *dD, void *ws,
                        cudaStream_t st);

// L > 16384 needs kgen_backward_workspace_bytes(H, L) of workspace (ws), else ws may be null
size_t kgen_backward_workspace_bytes(int H, int L);
cudaError_t launch_kgen_backward(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B,
                                 const float2 *C, const float *log_dt, const float *dK, int H, int Nh, int L,
                                 float2 *dLambda, float2 *dP, float2 *dQ, float2 *dB, float2 *dC,
                                 float *dlog_dt, void *ws, cudaStream_t st);

cudaError_t launch_irfft_packed(float *K, int H, int L, cudaStream_t st);
// K holds the packed half spectrum (k_cauchy's output) on entry and the kernel
// on exit; ws receives the spectrum of K + D delta_0 as launch_kspec leaves it
// (L = 16384: one fused launch; other L: launch_irfft_packed + launch_kspec)
cudaError_t launch_kspec_from_half(float *K, const float *D, int H, int L, void *ws, cudaStream_t st);

// ---- quad.cu: L = 16384 (a cluster of two CTAs holding four ranks) ----
cudaError_t launch_kspec_l16k(const float *K, const float *D, int H, void *ws, cudaStream_t st, const float *Ki);
cudaError_t launch_fftconv_l16k(const float *u, const void *ws, int Bt, int H, float *y, bool adjoint,
                                cudaStream_t st);
cudaError_t launch_kspec_from_half_l16k(float *K, const float *D, int H, void *ws, cudaStream_t st);

// ---- kgen.cu: K and the convolution spectrum of K + D delta_0 in one launch
// (L <= 8192; longer L runs k_cauchy, then launch_kspec_from_half) ----
cudaError_t launch_kgen(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B, const float2 *C,
                        const float *log_dt, const float *D, int H, int Nh, int L, float *K, void *ws,
                        unsigned *flags, cudaStream_t st);

// ---- cauchy.cu ----
cudaError_t launch_cauchy(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B,
                          const float2 *C, const float *log_dt, int H, int Nh, int L, float *K,
                          unsigned *flags, cudaStream_t st);

// ---- s4d.cu ----
cudaError_t launch_vandermonde(const float2 *A, const float2 *B, const float2 *C, const float *log_dt,
                               int H, int Nh, int L, float *K, unsigned *flags, cudaStream_t st);
cudaError_t launch_vandermonde_backward(const float2 *A, const float2 *B, const float2 *C, const float *log_dt,
                                        const float *dK, int H, int Nh, int L, float2 *dA, float2 *dB, float2 *dC,
                                        float *dlog_dt, cudaStream_t st);
cudaError_t launch_s4d_zoh(const float2 *A, const float2 *B, const float *log_dt, int H, int Nh,
                           float2 *Abar, float2 *Bbar, cudaStream_t st);

// ---- block.cu: the S4Block around the layer (norm, GLU projection, residual) ----
size_t glu_workspace_bytes(int H);
cudaError_t launch_layernorm_channels(const float *x, const float *gamma, const float *beta, float eps, int Bt,
                                      int H, int L, float *z, cudaStream_t st);
cudaError_t launch_glu_prepare(const float *W, int H, void *ws, cudaStream_t st);
cudaError_t launch_glu_projection(const float *y, const float *x, const float *bias, const void *ws, int Bt, int H,
                                  int L, float *out, unsigned *flags, cudaStream_t st);

// ---- zoh_dplr.cu: zero-order hold of the full DPLR system (Nh <= 32) ----
// K == nullptr: write Abar [H, N, N], Bbar [H, N], Cfull [H, N]; else the
// truncated kernel K [H, L]
cudaError_t launch_dplr_zoh(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B,
                            const float2 *C, const float *log_dt, int H, int Nh, int L, float2 *Abar,
                            float2 *Bbar, float2 *Cfull, float *K, unsigned *flags, cudaStream_t st);

// ---- decode.cu ----
cudaError_t launch_dplr_discretize(const float2 *Lambda, const float2 *P, const float2 *Q,
                                   const float2 *B, const float2 *C, const float *log_dt, int H, int Nh,
                                   float2 *Abar, float2 *Bbar, float2 *Cfull, cudaStream_t st);
cudaError_t launch_dplr_discretize_structured(const float2 *Lambda, const float2 *P, const float2 *Q,
                                              const float2 *B, const float *log_dt, int H, int Nh,
                                              float2 *Astr, float2 *Bbar, cudaStream_t st);
cudaError_t launch_dplr_ctilde(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *C,
                               const float *log_dt, int H, int Nh, int L, float2 *Ct, cudaStream_t st);
cudaError_t launch_step(int mode, const float2 *Abar, const float2 *Bbar, const float2 *C, const float *D,
                        int Bt, int H, int Ns, int T, float2 *x, const float *u, float *y, cudaStream_t st);

}  // namespace s4
