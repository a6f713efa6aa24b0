/*
 * s4dplr.h -- C ABI of libs4dplr.so: the S4 DPLR convolution kernel, the
 * zero-padded causal FFT convolution, the S4D Vandermonde kernel and the
 * recurrent (decode) step, on one NVIDIA B200 (sm_100a).
 *
 * Sources of the definitions (page title, section):
 *   [S4K] "The S4 kernel, from scratch": §1 The continuous state-space model,
 *         §3 Discretization, §4 The convolutional kernel via the generating
 *         function (and its "Aliasing" paragraph), §5 Two views, kept in sync,
 *         §6 Trainable layer.
 *   [S4W] "S4" (wiki page), section "S4D".
 *
 * Conventions shared by every entry point
 *   - All array pointers are DEVICE pointers unless stated otherwise. The
 *     caller allocates and owns every buffer; the library allocates no device
 *     memory and keeps no state between calls except per-device kernel
 *     attributes set once.
 *   - Arrays are row-major, last index contiguous. Complex numbers are pairs
 *     of float32 (re, im) -- the real (..., 2) storage of [S4K] §6.
 *   - Per-channel parameters of the H independent SSMs ([S4K] §1) are [H, Nh]:
 *     Nh stored modes. The system is conjugate-closed: each stored mode n has
 *     an implicit partner conj(mode n) (Lambda, P, Q, B and C all
 *     conjugated), so the full state size is N = 2 Nh and every kernel is real.
 *   - The step size enters as log_dt[h] (dt = exp(log_dt), [S4K] §6).
 *   - Every call is asynchronous on `stream` (0 = legacy default stream).
 *     Argument checks run on the host BEFORE anything is launched; on any
 *     error nothing is launched and the status says why. A failing CUDA launch
 *     returns S4_ERR_CUDA (see s4_last_cuda_error()).
 *   - Data-dependent conditions never trap: kernels OR bits into *d_flags
 *     (a device word; may be NULL), which the caller reads after a sync.
 *   - Calls on different streams may run concurrently as long as their
 *     output buffers (and workspaces) do not overlap.
 */
#ifndef S4DPLR_H
#define S4DPLR_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct { float re, im; } s4_c32; /* 8 bytes, 8-byte aligned */

typedef enum {
    S4_OK = 0,
    S4_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, overlap */
    S4_ERR_UNSUPPORTED = 2,  /* L not a power of two in [16, 65536], Nh > 256, ... */
    S4_ERR_WORKSPACE = 3,    /* workspace missing or smaller than the query says */
    S4_ERR_CUDA = 4          /* a CUDA runtime call or launch failed */
} s4_status;

/* Bits OR-ed into *d_flags by the kernels. */
#define S4_FLAG_UNSTABLE  1u  /* some Re(Lambda) >= 0 (or Re(a) >= 0 for S4D)   */
#define S4_FLAG_NONFINITE 2u  /* a non-finite value was produced                 */
#define S4_FLAG_TIMEOUT   4u  /* a bounded wait for the tensor cores ran out: the
                                 output is incomplete (not expected in practice) */

#define S4_MIN_L 16
#define S4_MAX_L 65536
#define S4_MAX_NH 256       /* stored modes per channel                          */
#define S4_MAX_H 65535      /* channels per call (kernel and decode entry points) */
#define S4_MAX_DENSE_N 128  /* full state size of the dense decode step           */

/* Human-readable name of a status code (static string, never NULL). */
const char *s4_status_string(s4_status s);

/* CUDA error code (cudaError_t as int) of the last S4_ERR_CUDA returned on
 * the calling host thread, 0 if none. */
int s4_last_cuda_error(void);

/* ABI version, currently 1. */
int s4_version(void);

/* ------------------------------------------------------------------------
 * s4_kernel_dplr -- the S4 convolution kernel K[H, L] of a bilinear-
 * discretised DPLR SSM ([S4K] §3 and §4).
 *
 * For each channel h, with dt = exp(log_dt[h]), A = Lambda - P Q^* and the
 * bilinear rule Abar = (I - dt/2 A)^-1 (I + dt/2 A), Bbar = (I - dt/2 A)^-1
 * dt B, Cbar = C, K is the ALIASED kernel ([S4K] §4 "Aliasing"):
 *     K[h, k] = sum_{p >= 0} Cbar Abar^(k + pL) Bbar,   k = 0 .. L-1,
 * computed as in [S4K] §4: the generating function is evaluated at the L-th
 * roots of unity z_j = exp(-2 pi i j / L) by four Cauchy sums over the modes
 * (k00, k01, k10, k11), the rank-1 Woodbury correction and the factor
 * 2/(1+z); a length-L inverse FFT then gives K. Only j = 0 .. L/2 are
 * evaluated (conjugate symmetry); j = L/2 (z = -1) uses the limit
 * dt * Re sum_n C_n B_n.
 *
 *   Lambda, P, Q, B, C : [H, Nh] complex, device, 8-byte aligned. Q enters as
 *                        conj(Q) in k10 and k11 (A = Lambda - P Q^*).
 *   log_dt             : [H] float, device.
 *   1 <= H <= 65535, 1 <= Nh <= 256, L a power of two in [16, 65536].
 *   K                  : [H, L] float out, device, 16-byte aligned. It is also
 *                        used as scratch (the half spectrum is staged in it).
 *   d_flags            : device unsigned or NULL; S4_FLAG_UNSTABLE if some
 *                        Re(Lambda) >= 0 (K is still computed),
 *                        S4_FLAG_NONFINITE if a spectrum value is not finite.
 * Errors: S4_ERR_INVALID_ARG (null, H < 1, Nh < 1, misaligned),
 *         S4_ERR_UNSUPPORTED (L or Nh out of range), S4_ERR_CUDA.
 * ------------------------------------------------------------------------ */
s4_status s4_kernel_dplr(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                         const s4_c32 *B, const s4_c32 *C, const float *log_dt,
                         int H, int Nh, int L, float *K, unsigned *d_flags,
                         cudaStream_t stream);

/* s4_kernel_dplr in two halves (the kernels it runs, in order):
 * s4_dplr_spectrum writes the generating function at j = 0 .. L/2, times
 * 1/L, packed into K[h, :] as K[h,0] = K_hat_0 (real), K[h,1] = K_hat_{L/2}
 * (real), K[h,2j], K[h,2j+1] = Re, Im K_hat_j for 0 < j < L/2 ([S4K] §4,
 * the four Cauchy sums, Woodbury and 2/(1+z)); s4_irfft_packed turns such a
 * packed half spectrum into the real kernel, in place ([S4K] §4, "an inverse
 * FFT returns the time-domain kernel"). Same argument rules as s4_kernel_dplr. */
s4_status s4_dplr_spectrum(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                           const s4_c32 *B, const s4_c32 *C, const float *log_dt,
                           int H, int Nh, int L, float *K, unsigned *d_flags,
                           cudaStream_t stream);
s4_status s4_irfft_packed(float *K, int H, int L, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * s4_fft_conv -- y = K * u + D u along the last axis, causal, for every row
 * (b, h) ([S4K] §1 for y = Cx + Du, §5 "fft_conv", zero-padded so the
 * circular FFT product has no wrap-around):
 *     y[b, h, t] = sum_{s=0}^{t} K[h, s] u[b, h, t - s] + D[h] u[b, h, t].
 * Computed with length-2L transforms (input zero-padded to 2L, output
 * cropped to [0, L)). Two rows of the same channel are transformed together
 * as one complex signal.
 *
 *   u : [Bt, H, L] float, device, 16-byte aligned.   K : [H, L] float, device,
 *   16-byte aligned.   D : [H] float, device.   y : [Bt, H, L] float out,
 *   device, 16-byte aligned, must not overlap u, K, D or the workspace.
 *   Bt, H >= 1; L a power of two in [16, 65536]; Bt*H*L < 2^40.
 *   workspace : device, 256-byte aligned, at least
 *               s4_fft_conv_workspace_size(H, L) bytes (H * 2L complex
 *               floats, rounded up to 256 bytes); holds the spectrum of the
 *               zero-padded K + D delta_0 after the call.
 * Errors: S4_ERR_INVALID_ARG, S4_ERR_UNSUPPORTED, S4_ERR_WORKSPACE, S4_ERR_CUDA.
 * ------------------------------------------------------------------------ */
s4_status s4_fft_conv_workspace_size(int H, int L, size_t *bytes);

s4_status s4_fft_conv(const float *u, const float *K, const float *D,
                      int Bt, int H, int L, float *y,
                      void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* s4_fft_conv in two halves, for callers that apply one kernel to many
 * batches: _prepare writes into the workspace the spectrum of the
 * zero-padded K + D delta_0 (so the D u term comes out of the same product);
 * _apply convolves u with that spectrum. s4_fft_conv(...) == _prepare(K, D)
 * then _apply(u). In _prepare, D may be NULL (no feed-through term). The
 * workspace must come from a _prepare with the same H and L and must not be
 * written in between; other rules as for s4_fft_conv. */
s4_status s4_fft_conv_prepare(const float *K, const float *D, int H, int L,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream);
s4_status s4_fft_conv_apply(const float *u, const void *workspace,
                            int Bt, int H, int L, float *y,
                            size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Backward pass of the convolution ([S4K] §5 fft_conv; §6 trains the layer):
 * for y = K * u + D u and an upstream gradient dy [Bt, H, L],
 *
 * s4_fft_conv_apply_adjoint: du = dL/du, the correlation
 *     du[b,h,s] = sum_{t>=s} K[h,t-s] dy[b,h,t] + D[h] dy[b,h,s],
 *   with the same workspace as s4_fft_conv_apply (from s4_fft_conv_prepare or
 *   s4_kernel_dplr_prepare): the forward kernel with the conjugate spectrum.
 *   Arguments and errors as s4_fft_conv_apply (dy in place of u, du of y).
 *
 * s4_fft_conv_kernel_grad: dK = dL/dK [H, L] and dD = dL/dD [H],
 *     dK[h,k] = sum_b sum_{t>=k} dy[b,h,t] u[b,h,t-k],   dD[h] = dK[h,0].
 *   u, dy [Bt, H, L] device, 16-byte aligned; dK [H, L] out, 16-byte
 *   aligned; dD [H] out, nullable. Workspace:
 *   s4_fft_conv_kernel_grad_workspace_size bytes, 256-byte aligned,
 *   caller-owned, contents irrelevant on entry. L <= 8192: 2 H 2L 8 bytes (a
 *   per-channel accumulator of the spectrum products and a per-channel
 *   scratch; one launch). L > 8192: the convolution workspace of (H, L) plus
 *   2 H L 4 bytes; per pair of batch rows the spectrum of the zero-padded
 *   complex signal u[b] + i u[b+1] is prepared as if it were a kernel
 *   spectrum, and the real part of the adjoint convolution of dy[b], dy[b+1]
 *   with it is the two rows' share of dK (3 launches per row pair). Either
 *   way the rows are summed in a fixed order (deterministic).
 *   Errors: null pointers, Bt/H < 1, misalignment, overlapping buffers ->
 *   S4_ERR_INVALID_ARG; workspace too small or misaligned ->
 *   S4_ERR_WORKSPACE.
 * ------------------------------------------------------------------------ */
s4_status s4_fft_conv_apply_adjoint(const float *dy, const void *workspace,
                                    int Bt, int H, int L, float *du,
                                    size_t workspace_bytes, cudaStream_t stream);

s4_status s4_fft_conv_kernel_grad_workspace_size(int H, int L, size_t *bytes);

s4_status s4_fft_conv_kernel_grad(const float *u, const float *dy, int Bt, int H, int L,
                                  float *dK, float *dD, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * s4_kernel_dplr_backward: the gradient of a loss through the DPLR kernel
 * ([S4K] §4 generating function; §6 trains Lambda, P, Q, B, C and log dt)
 * with respect to the parameters, given dK = dLoss/dK [H, L] (for instance
 * from s4_fft_conv_kernel_grad). For each complex parameter the result is
 * dLoss/dRe + i dLoss/dIm of the stored modes (the implicit conjugate modes
 * are accounted for); dlog_dt is the derivative in log dt. The gradient runs
 * through DFT(dK) at the same roots of unity and the derivatives of the
 * four Cauchy sums, the Woodbury correction and the bilinear factor
 * (squared-denominator Cauchy sums for Lambda and dt), and the closed form at
 * the Nyquist bin. s4_kernel_dplr_backward: L <= 16384 (longer ->
 * S4_ERR_UNSUPPORTED). s4_kernel_dplr_backward_ws: any L; for L > 16384
 * DFT(dK) is formed by a four-step transform (L = 256 x L/256) in the
 * workspace (s4_kernel_dplr_backward_workspace_size bytes: H L 8 + H (L/2+1) 8,
 * each rounded up to 256; 0 for L <= 16384, where the workspace may be NULL),
 * 256-byte aligned, caller-owned, not overlapping the outputs or dK.
 *   Lambda, P, Q, B, C : [H, Nh] complex;  log_dt : [H];  dK : [H, L].
 *   dLambda, dP, dQ, dB, dC : [H, Nh] complex out;  dlog_dt : [H] out.
 * Errors: null pointers, misaligned complex arrays, outputs overlapping
 * inputs or each other -> S4_ERR_INVALID_ARG; L not a power of two in range,
 * Nh > S4_MAX_NH -> S4_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------ */
s4_status s4_kernel_dplr_backward(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                                  const s4_c32 *B, const s4_c32 *C, const float *log_dt,
                                  const float *dK, int H, int Nh, int L, s4_c32 *dLambda,
                                  s4_c32 *dP, s4_c32 *dQ, s4_c32 *dB, s4_c32 *dC,
                                  float *dlog_dt, cudaStream_t stream);

s4_status s4_kernel_dplr_backward_workspace_size(int H, int L, size_t *bytes);

s4_status s4_kernel_dplr_backward_ws(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                                     const s4_c32 *B, const s4_c32 *C, const float *log_dt,
                                     const float *dK, int H, int Nh, int L, s4_c32 *dLambda,
                                     s4_c32 *dP, s4_c32 *dQ, s4_c32 *dB, s4_c32 *dC,
                                     float *dlog_dt, void *workspace, size_t workspace_bytes,
                                     cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The whole forward pass of the layer's convolution view ([S4K] §4, §5).
 *
 * s4_kernel_dplr_prepare = s4_kernel_dplr(...) followed by
 * s4_fft_conv_prepare(K, D, ...): it writes K[H, L] and the convolution
 * spectrum of K + D delta_0 into the workspace. For L <= 8192 both come out
 * of a single kernel per channel (the generating function is written
 * straight into the inverse transform's input order, and the inverse
 * transform's output starts the zero-padded forward transform); for
 * L = 16384 the Cauchy stage is one launch and the inverse transform, K and
 * the spectrum a second (K is stored, never read back); longer L run the
 * Cauchy stage, the inverse transform and the spectrum as three launches.
 * D may be NULL (no feed-through term).
 *
 * s4_forward_dplr = s4_kernel_dplr_prepare followed by s4_fft_conv_apply:
 * y[Bt, H, L] from the DPLR parameters and u in one call; K and the
 * workspace are outputs/scratch as above. Argument rules and errors are those
 * of the calls it is made of (D required here).
 * ------------------------------------------------------------------------ */
s4_status s4_kernel_dplr_prepare(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                                 const s4_c32 *B, const s4_c32 *C, const float *log_dt,
                                 const float *D, int H, int Nh, int L, float *K,
                                 void *workspace, size_t workspace_bytes, unsigned *d_flags,
                                 cudaStream_t stream);

s4_status s4_forward_dplr(const float *u, const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                          const s4_c32 *B, const s4_c32 *C, const float *log_dt, const float *D,
                          int Bt, int H, int Nh, int L, float *K, float *y,
                          void *workspace, size_t workspace_bytes, unsigned *d_flags,
                          cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Host-buffer forms: s4_fft_conv and s4_forward_dplr with u and y in HOST
 * memory, the copies pipelined with the convolution. The batch is cut into
 * nchunks chunks of whole row pairs (when it has fewer row pairs than
 * nchunks and L <= 16384, into row pairs cut into channel slices, so that a
 * small batch still pipelines); chunk c is uploaded on h2d_stream,
 * convolved on `stream` once it has arrived, and downloaded on d2h_stream
 * once convolved, so the upload of one chunk, the convolution of the next
 * earlier one and the download of the one before overlap (the two copy
 * directions run on separate copy engines). The kernel spectrum
 * (s4_fft_conv_host) or the kernel generation (s4_forward_dplr_host) runs
 * on `stream` first, overlapping the first upload. The uploads wait for the
 * work already queued on `stream`; `stream` waits for the last download, so
 * synchronising `stream` completes y_host. Results equal those of the
 * device-buffer forms.
 *   u_host, y_host : [Bt, H, L] host memory; page-locked memory
 *                    (cudaHostAlloc, cudaHostRegister) lets the copies run
 *                    asynchronously and overlap, pageable memory still works.
 *   u_dev, y_dev   : [Bt, H, L] device staging buffers owned by the caller
 *                    (16-byte aligned, not overlapping each other, K, D,
 *                    the workspace or the parameters); what they hold on
 *                    return is staging data in the chunks' own order, not a
 *                    copy of u or y.
 *   nchunks        : >= 1 (clamped to the number of row pairs). Every
 *                    copy has a fixed cost on the PCIe link, so a few large
 *                    chunks beat many small ones: on a B200 at
 *                    Bt*H*L = 2^25 floats, 2 to 4 chunks ran fastest and 32
 *                    or more cost 20 to 45 % more per call.
 *   h2d_stream, d2h_stream : caller-owned streams (may be `stream` itself,
 *                    which serialises the pipeline).
 * Calls on different `stream`s, each with its own staging buffers,
 * workspace and K, may be in flight together: with shared copy streams one
 * call's downloads then overlap the next call's uploads, which removes the
 * pipeline's fill and drain from all but the first and last call.
 * The first call on each (host thread, device) creates the few CUDA events
 * the pipeline orders itself with, and later calls from that thread reuse
 * them (they live until the process exits); no call allocates memory.
 * Errors: as the device-buffer forms; null host pointers, overlapping host
 * buffers or nchunks < 1 -> S4_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------ */
s4_status s4_fft_conv_host(const float *u_host, const float *K, const float *D, int Bt, int H, int L,
                           float *y_host, float *u_dev, float *y_dev, void *workspace,
                           size_t workspace_bytes, int nchunks, cudaStream_t stream,
                           cudaStream_t h2d_stream, cudaStream_t d2h_stream);

s4_status s4_forward_dplr_host(const float *u_host, const s4_c32 *Lambda, const s4_c32 *P,
                               const s4_c32 *Q, const s4_c32 *B, const s4_c32 *C,
                               const float *log_dt, const float *D, int Bt, int H, int Nh, int L,
                               float *y_host, float *K, float *u_dev, float *y_dev, void *workspace,
                               size_t workspace_bytes, unsigned *d_flags, int nchunks,
                               cudaStream_t stream, cudaStream_t h2d_stream,
                               cudaStream_t d2h_stream);

/* ------------------------------------------------------------------------
 * s4_fft_conv_static -- s4_fft_conv without a caller-provided workspace.
 * The pages have no counterpart of this entry point; it exists for callers
 * that cannot allocate device memory: a plugin inside a host application
 * whose memory pool owns the GPU, or a real-time path where cudaMalloc's
 * implicit device synchronisation is not allowed. It allocates nothing.
 *
 * The workspace is a library-owned device array of S4_STATIC_SCRATCH_BYTES
 * (32 MiB); every GPU that loads the library keeps it until the process
 * exits. The first call on a device looks up that array's device address
 * (with that device current), so make the first call on each device before
 * any stream capture. All calls share the one array: calls that overlap on
 * the GPU (other streams, other host threads) race on it and must be
 * serialised by the caller. Each call overwrites all the scratch it reads, so
 * nothing in it has to start at zero.
 *
 * Arguments, layouts and errors are those of s4_fft_conv; in addition the
 * call returns S4_ERR_UNSUPPORTED when s4_fft_conv_workspace_size(H, L)
 * exceeds S4_STATIC_SCRATCH_BYTES (about H * L <= 2 M elements), and
 * S4_ERR_INVALID_ARG when u, K, D or y is not memory the current device can
 * address as its own (a device buffer of another GPU, or unregistered host
 * memory): the scratch used is the current device's.
 * ------------------------------------------------------------------------ */
#define S4_STATIC_SCRATCH_BYTES (32u << 20)

s4_status s4_fft_conv_static(const float *u, const float *K, const float *D,
                             int Bt, int H, int L, float *y, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Zero-order hold of the DPLR system ([S4K] §3: the ZOH rule, applied here to
 * the dense matrix of the full conjugate-closed system A = diag(Lambda_f) -
 * P_f Q_f^*, N = 2 Nh):
 *     Abar = exp(dt A),  Bbar = (integral_0^dt exp(A s) ds) B_f,  Cbar = C_f.
 * The generating-function shortcut of [S4K] §4 is specific to the bilinear
 * rule, so under ZOH the kernel is formed from dense powers:
 *     K[h, k] = Re(C_f Abar^k Bbar),  k = 0 .. L-1  (TRUNCATED: no aliasing).
 * Computed per channel in fp64 (scaling and squaring of the augmented
 * exponential, Taylor degree 16), results rounded to fp32.
 *
 * s4_dplr_discretize_zoh: Abar [H, N, N], Bbar [H, N], Cfull [H, N] out --
 *   the layout of s4_dplr_discretize, so the dense recurrent step
 *   (S4_STEP_DENSE) runs the ZOH system unchanged.
 * s4_kernel_dplr_zoh: K [H, L] out (16-byte aligned); d_flags (nullable):
 *   S4_FLAG_UNSTABLE if some Re(Lambda) >= 0, S4_FLAG_NONFINITE if a kernel
 *   value is not finite. K then feeds s4_fft_conv_prepare like any kernel.
 * Both: Lambda, P, Q, B, C [H, Nh] complex, log_dt [H]; 1 <= Nh <= 32
 * (larger -> S4_ERR_UNSUPPORTED); L a power of two in [16, 65536]. Errors as
 * s4_dplr_discretize / s4_kernel_dplr.
 * ------------------------------------------------------------------------ */
#define S4_MAX_ZOH_NH 32

s4_status s4_dplr_discretize_zoh(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                                 const s4_c32 *B, const s4_c32 *C, const float *log_dt, int H,
                                 int Nh, s4_c32 *Abar, s4_c32 *Bbar, s4_c32 *Cfull,
                                 cudaStream_t stream);

s4_status s4_kernel_dplr_zoh(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                             const s4_c32 *B, const s4_c32 *C, const float *log_dt, int H,
                             int Nh, int L, float *K, unsigned *d_flags, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The S4Block around the layer ([S4K] §6 "Trainable layer": a pre-norm, a
 * GLU-gated projection and a residual connection). All tensors [Bt, H, L]
 * float, device, 16-byte aligned, time (L) contiguous -- the layout of u and
 * y above. 1 <= Bt, 1 <= H <= 8192, L a power of two in [16, 65536],
 * Bt * H * L < 2^40.
 *
 * s4_layernorm_channels: z[b,h,t] = (x[b,h,t] - mu[b,t]) / sqrt(var[b,t] +
 *   eps) * gamma[h] + beta[h], mu and var the mean and the biased variance
 *   of x[b, :, t] over the H channels. gamma, beta: [H] device. eps > 0.
 *   z may equal x (in place) but must not otherwise overlap it.
 *
 * s4_glu_projection_prepare: splits W [2H, H] (device; rows [0, H) give the
 *   GLU value, rows [H, 2H) the gate) into the operand images the projection
 *   reads: bf16 high and low parts of every weight, laid out for the tensor
 *   cores. workspace: s4_glu_projection_workspace_size(H) bytes, device,
 *   256-byte aligned, caller-owned; valid until W changes.
 *
 * s4_glu_projection_residual: out[b,o,t] = x[b,o,t] + p[o] * sigmoid(p[H+o]),
 *   p = W y[b, :, t] + bias, with W from the prepared workspace and bias
 *   [2H] device. The product runs on the tensor cores as three bf16 products
 *   of the split operands with fp32 accumulation (relative error ~1e-5 of
 *   the sum of |W||y| terms). out may equal x; out must not overlap y or the
 *   workspace. d_flags (nullable): S4_FLAG_TIMEOUT if a bounded wait for the
 *   tensor cores ran out (the output is then incomplete).
 *
 * s4_block_forward: out = x + GLU(W S4(LN(x)) + bias) in three launches:
 *   s4_layernorm_channels(x) -> z, s4_fft_conv_apply(z) -> y with the
 *   prepared convolution workspace of the layer (s4_fft_conv_prepare or
 *   s4_kernel_dplr_prepare: the spectrum of K + D delta_0), then
 *   s4_glu_projection_residual(y, x) -> out. z and y are caller-owned
 *   [Bt, H, L] buffers (they are the activations a backward pass needs);
 *   out may equal x.
 *
 * Errors: null pointers, H > 8192, Bt/H < 1, eps <= 0 or not finite,
 * misalignment, forbidden overlaps -> S4_ERR_INVALID_ARG; L not a power of
 * two in range -> S4_ERR_UNSUPPORTED; workspace too small or misaligned ->
 * S4_ERR_WORKSPACE.
 * ------------------------------------------------------------------------ */
#define S4_MAX_BLOCK_H 8192

s4_status s4_layernorm_channels(const float *x, const float *gamma, const float *beta, float eps,
                                int Bt, int H, int L, float *z, cudaStream_t stream);

s4_status s4_glu_projection_workspace_size(int H, size_t *bytes);

s4_status s4_glu_projection_prepare(const float *W, int H, void *workspace, size_t workspace_bytes,
                                    cudaStream_t stream);

s4_status s4_glu_projection_residual(const float *y, const float *x, const float *bias,
                                     const void *workspace, size_t workspace_bytes,
                                     int Bt, int H, int L, float *out, unsigned *d_flags,
                                     cudaStream_t stream);

s4_status s4_block_forward(const float *x, const float *gamma, const float *beta, float eps,
                           const void *conv_workspace, size_t conv_workspace_bytes,
                           const float *bias, const void *glu_workspace, size_t glu_workspace_bytes,
                           int Bt, int H, int L, float *z, float *y, float *out, unsigned *d_flags,
                           cudaStream_t stream);

/* ------------------------------------------------------------------------
 * s4d_kernel_vandermonde -- kernel of the diagonal S4D SSM with zero-order
 * hold ([S4W] "S4D"; ZOH rule of [S4K] §3):
 *     Abar_n = exp(dt a_n),  Bbar_n = (exp(dt a_n) - 1)/a_n * B_n,
 *     K[h, k] = 2 Re sum_{n < Nh} C_n Bbar_n Abar_n^k,   k = 0 .. L-1
 * (the TRUNCATED kernel: no aliasing). Powers are formed from fp64 phase
 * reductions, so long kernels keep their phase accuracy.
 *
 *   A, B, C : [H, Nh] complex, device (A holds the continuous-time a_n).
 *   log_dt  : [H] float.  K : [H, L] float out, 16-byte aligned.
 *   1 <= H <= 65535, 1 <= Nh <= 256, L a power of two in [16, 65536].
 *   d_flags : as above (S4_FLAG_UNSTABLE if some Re(a_n) >= 0).
 * ------------------------------------------------------------------------ */
s4_status s4d_kernel_vandermonde(const s4_c32 *A, const s4_c32 *B, const s4_c32 *C,
                                 const float *log_dt, int H, int Nh, int L, float *K,
                                 unsigned *d_flags, cudaStream_t stream);

/* s4d_kernel_vandermonde_backward: the gradient of a loss through the S4D
 * kernel ([S4W] "S4D"; the layer is trained as in [S4K] §6) given
 * dK = dLoss/dK [H, L]: dA, dB, dC [H, Nh] complex out as dLoss/dRe +
 * i dLoss/dIm of each stored mode (its conjugate partner accounted for), and
 * dlog_dt [H] out. With V_n = sum_k dK[k] Abar_n^k, W_n = sum_k k dK[k]
 * Abar_n^k and r_n = (exp(dt a_n) - 1)/a_n:
 *   dC = 2 conj(Bbar V), dB = 2 conj(C r V),
 *   dA = 2 conj(C B dt^2 phi1'(dt a) V + C Bbar dt W), phi1(x) = (e^x - 1)/x,
 *   dlog_dt = 2 dt Re sum_n (C B Abar V + C Bbar a W).
 * V, W are summed over 64-step blocks whose first power is evaluated
 * directly (fp64 phase reduction); fp64 accumulation across blocks.
 * Any L (power of two in [16, 65536]), Nh <= 256. Errors: null pointers,
 * misaligned complex arrays, outputs overlapping inputs or each other ->
 * S4_ERR_INVALID_ARG; bad L, Nh -> S4_ERR_UNSUPPORTED. */
s4_status s4d_kernel_vandermonde_backward(const s4_c32 *A, const s4_c32 *B, const s4_c32 *C,
                                          const float *log_dt, const float *dK, int H, int Nh,
                                          int L, s4_c32 *dA, s4_c32 *dB, s4_c32 *dC,
                                          float *dlog_dt, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Decode set-up ([S4K] §3 and §5, recurrent view).
 *
 * s4_dplr_discretize: dense bilinear discretisation of the full
 * conjugate-closed DPLR system (N = 2 Nh modes, stored modes first, then
 * their conjugates): A = diag(Lambda_f) - P_f Q_f^*,
 *     Abar = (I - dt/2 A)^-1 (I + dt/2 A),   Bbar = (I - dt/2 A)^-1 dt B_f,
 *     Cfull = C_f.
 * The inverse uses the Sherman-Morrison form of the diagonal-plus-rank-1
 * matrix I - dt/2 A.
 *   Abar : [H, N, N] complex out; Bbar, Cfull : [H, N] complex out.
 *
 * s4d_discretize_zoh: S4D diagonal ZOH, Abar[h, n] = exp(dt a_n),
 * Bbar[h, n] = (exp(dt a_n) - 1)/a_n B_n ([S4K] §3 ZOH; cancellation-free
 * expm1). Abar, Bbar : [H, Nh] complex out.
 * ------------------------------------------------------------------------ */
s4_status s4_dplr_discretize(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                             const s4_c32 *B, const s4_c32 *C, const float *log_dt,
                             int H, int Nh, s4_c32 *Abar, s4_c32 *Bbar, s4_c32 *Cfull,
                             cudaStream_t stream);

s4_status s4d_discretize_zoh(const s4_c32 *A, const s4_c32 *B, const float *log_dt,
                             int H, int Nh, s4_c32 *Abar, s4_c32 *Bbar,
                             cudaStream_t stream);

/* ------------------------------------------------------------------------
 * s4_dplr_ctilde: Ctilde = C (I - Abar^L) over the full conjugate-closed
 * bilinear system (Abar as s4_dplr_discretize). The generating function at
 * the L-th roots of unity gives the aliased kernel sum_p K_{k + pL}
 * ([S4K] §4, "Aliasing"); with Ctilde in place of C, s4_kernel_dplr (and
 * s4_forward_dplr) return the truncated kernel Cbar Abar^k Bbar, k < L,
 * whose convolution equals the recurrence from a zero state exactly.
 * c = C_f is carried through L products c <- c Abar in the structured form
 * of s4_dplr_discretize_structured, in fp64 (O(L Nh) per channel, one warp
 * per channel; a one-time reparameterisation, not a per-step cost).
 *   Lambda, P, Q, C : [H, Nh] complex; log_dt : [H]; L >= 1.
 *   Ctilde : [H, Nh] complex out (stored half); may not alias the inputs.
 * Errors: null pointers, L < 1, H or Nh < 1 -> S4_ERR_INVALID_ARG;
 * Nh > S4_MAX_NH or H > S4_MAX_H -> S4_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------ */
s4_status s4_dplr_ctilde(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *C,
                         const float *log_dt, int H, int Nh, int L, s4_c32 *Ctilde,
                         cudaStream_t stream);

/* ------------------------------------------------------------------------
 * s4_dplr_discretize_structured: the same bilinear DPLR discretisation
 * ([S4K] §3 rule on the §2 DPLR system) kept in its diagonal-plus-rank-1
 * form, for the O(Nh) step S4_STEP_DPLR ([S4K] §5 recurrent view). With
 * d_n = 1 - dt/2 Lambda_n, alpha_n = (dt/2) P_n / d_n, beta_n = conj(Q_n)/d_n
 * and s = 1 + 2 Re sum_n conj(Q_n) alpha_n (the Sherman-Morrison denominator
 * of I - dt/2 A over the full conjugate-closed system),
 *     Abar = diag(a) - g beta^T,  a_n = 2/d_n - 1,  g_n = 2 alpha_n / s,
 * over the full system; only the stored half is written:
 *   Astr : [H, Nh, 3] complex out, Astr[h, n] = {a_n, g_n, beta_n};
 *   Bbar : [H, Nh] complex out, the stored half of s4_dplr_discretize's Bbar.
 * Computed in fp64, stored as fp32. Errors as s4_dplr_discretize.
 * ------------------------------------------------------------------------ */
s4_status s4_dplr_discretize_structured(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                                        const s4_c32 *B, const float *log_dt, int H, int Nh,
                                        s4_c32 *Astr, s4_c32 *Bbar, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * s4_recurrent_step -- one token of the recurrence ([S4K] §5):
 *     x <- Abar x + Bbar u_t,   y_t = Re(C . x) + D u_t        (dense)
 *     x <- Abar * x + Bbar u_t, y_t = 2 Re(sum_n C_n x_n) + D u_t  (diagonal)
 * The state x is owned by the caller (a nonzero initial state is allowed).
 *   mode S4_STEP_DENSE: Abar [H, Ns, Ns], Bbar, C [H, Ns] with Ns = N = 2 Nh
 *                       (from s4_dplr_discretize), Ns <= 128 (Abar of a
 *                       channel is staged in shared memory).
 *   mode S4_STEP_DIAG : Abar, Bbar, C [H, Ns] with Ns = Nh (S4D), Ns <= 256.
 *   mode S4_STEP_DPLR : structured DPLR step, O(Nh) per token: Abar = Astr
 *                       [H, Ns, 3] and Bbar [H, Ns] from
 *                       s4_dplr_discretize_structured, C [H, Ns] (stored
 *                       modes), Ns = Nh <= 256. x holds the stored half of a
 *                       conjugate-symmetric full state (zero, for instance;
 *                       real inputs keep it so), and
 *                       y_t = 2 Re(sum_n C_n x_n) + D u_t, which equals the
 *                       dense step's Re(Cfull . x_full).
 *   x   : [Bt, H, Ns] complex in/out.   u_t, y_t : [Bt, H] float.  D : [H].
 *   1 <= H <= 65535; Bt >= 1.
 * s4_recurrent_scan runs T consecutive steps in one launch:
 *   u, y : [Bt, H, T] float (token axis last), x in/out as above.
 * ------------------------------------------------------------------------ */
typedef enum { S4_STEP_DENSE = 0, S4_STEP_DIAG = 1, S4_STEP_DPLR = 2 } s4_step_mode;

s4_status s4_recurrent_step(s4_step_mode mode, const s4_c32 *Abar, const s4_c32 *Bbar,
                            const s4_c32 *C, const float *D, int Bt, int H, int Ns,
                            s4_c32 *x, const float *u_t, float *y_t, cudaStream_t stream);

s4_status s4_recurrent_scan(s4_step_mode mode, const s4_c32 *Abar, const s4_c32 *Bbar,
                            const s4_c32 *C, const float *D, int Bt, int H, int Ns, int T,
                            s4_c32 *x, const float *u, float *y, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* S4DPLR_H */
