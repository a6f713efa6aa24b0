// api.cu -- the extern "C" entry points of libs4dplr.so (declared and
// documented in include/s4dplr.h). Every argument is checked on the host
// before anything is launched; nothing here allocates device memory.
#include <cstdint>

#include "launch.h"
#include "s4dplr.h"

namespace {

thread_local int g_last_cuda_error = 0;

s4_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return S4_OK;
    g_last_cuda_error = (int)e;
    return S4_ERR_CUDA;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool pow2_L(int L) { return L >= S4_MIN_L && L <= S4_MAX_L && (L & (L - 1)) == 0; }

bool overlap(const void *a, size_t an, const void *b, size_t bn) {
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + bn && y < x + an;
}

// common checks of the DPLR / S4D parameter sets
s4_status check_modes(int H, int Nh, int L, bool need_L) {
    if (H < 1 || Nh < 1) return S4_ERR_INVALID_ARG;
    if (Nh > S4_MAX_NH || H > S4_MAX_H) return S4_ERR_UNSUPPORTED;
    if (need_L && !pow2_L(L)) return S4_ERR_UNSUPPORTED;
    return S4_OK;
}

template <class... T>
bool any_null(const T *...p) { return ((p == nullptr) || ...); }

bool params_aligned(std::initializer_list<const void *> ps) {
    for (const void *p : ps)
        if (!aligned(p, 8)) return false;
    return true;
}

s4_status conv_checks(const float *u, int Bt, int H, int L, const float *y, const void *ws, size_t ws_bytes) {
    if (any_null(u, y) || ws == nullptr) return S4_ERR_INVALID_ARG;
    if (Bt < 1 || H < 1) return S4_ERR_INVALID_ARG;
    if (!pow2_L(L)) return S4_ERR_UNSUPPORTED;
    if ((double)Bt * (double)H * (double)L >= 1099511627776.0) return S4_ERR_INVALID_ARG;   // 2^40
    if (!aligned(u, 16) || !aligned(y, 16)) return S4_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return S4_ERR_WORKSPACE;
    if (ws_bytes < s4::conv_workspace_bytes(H, L)) return S4_ERR_WORKSPACE;
    const size_t nb = (size_t)Bt * H * L * sizeof(float);
    if (overlap(u, nb, y, nb) || overlap(y, nb, ws, ws_bytes)) return S4_ERR_INVALID_ARG;
    return S4_OK;
}

s4_status prepare_checks(const float *K, const float *D, int H, int L, const void *ws, size_t ws_bytes) {
    if (K == nullptr || ws == nullptr || H < 1) return S4_ERR_INVALID_ARG;
    if (!pow2_L(L)) return S4_ERR_UNSUPPORTED;
    if (!aligned(K, 16) || !aligned(D, 4)) return S4_ERR_INVALID_ARG;
    if (!aligned(ws, 256) || ws_bytes < s4::conv_workspace_bytes(H, L)) return S4_ERR_WORKSPACE;
    if (overlap(K, (size_t)H * L * sizeof(float), ws, ws_bytes)) return S4_ERR_INVALID_ARG;
    if (D != nullptr && overlap(D, (size_t)H * sizeof(float), ws, ws_bytes)) return S4_ERR_INVALID_ARG;
    return S4_OK;
}

}  // namespace

void s4::record_cuda_error(cudaError_t e) { g_last_cuda_error = (int)e; }

extern "C" {

const char *s4_status_string(s4_status s) {
    switch (s) {
        case S4_OK: return "S4_OK";
        case S4_ERR_INVALID_ARG: return "S4_ERR_INVALID_ARG";
        case S4_ERR_UNSUPPORTED: return "S4_ERR_UNSUPPORTED";
        case S4_ERR_WORKSPACE: return "S4_ERR_WORKSPACE";
        case S4_ERR_CUDA: return "S4_ERR_CUDA";
        default: return "S4_ERR_UNKNOWN";
    }
}

int s4_last_cuda_error(void) { return g_last_cuda_error; }

int s4_version(void) { return 1; }

static s4_status dplr_checks(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                             const s4_c32 *C, const float *log_dt, int H, int Nh, int L, const float *K) {
    if (any_null(Lambda, P, Q, B, C) || log_dt == nullptr || K == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, L, true);
    if (s != S4_OK) return s;
    if (!params_aligned({Lambda, P, Q, B, C}) || !aligned(K, 16) || !aligned(log_dt, 4))
        return S4_ERR_INVALID_ARG;
    const size_t kb = (size_t)H * L * sizeof(float), pb = (size_t)H * Nh * sizeof(s4_c32);
    for (const void *p : {(const void *)Lambda, (const void *)P, (const void *)Q, (const void *)B,
                          (const void *)C})
        if (overlap(K, kb, p, pb)) return S4_ERR_INVALID_ARG;
    if (overlap(K, kb, log_dt, (size_t)H * sizeof(float))) return S4_ERR_INVALID_ARG;
    return S4_OK;
}

s4_status s4_dplr_spectrum(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                           const s4_c32 *C, const float *log_dt, int H, int Nh, int L, float *K,
                           unsigned *d_flags, cudaStream_t stream) {
    s4_status s = dplr_checks(Lambda, P, Q, B, C, log_dt, H, Nh, L, K);
    if (s != S4_OK) return s;
    return cuda_status(s4::launch_cauchy((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q,
                                         (const float2 *)B, (const float2 *)C, log_dt, H, Nh, L, K, d_flags,
                                         stream));
}

s4_status s4_irfft_packed(float *K, int H, int L, cudaStream_t stream) {
    if (K == nullptr || H < 1) return S4_ERR_INVALID_ARG;
    if (H > S4_MAX_H || !pow2_L(L)) return S4_ERR_UNSUPPORTED;
    if (!aligned(K, 16)) return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_irfft_packed(K, H, L, stream));
}

s4_status s4_kernel_dplr(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                         const s4_c32 *C, const float *log_dt, int H, int Nh, int L, float *K,
                         unsigned *d_flags, cudaStream_t stream) {
    s4_status s = dplr_checks(Lambda, P, Q, B, C, log_dt, H, Nh, L, K);
    if (s != S4_OK) return s;
    cudaError_t e = s4::launch_cauchy((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q,
                                      (const float2 *)B, (const float2 *)C, log_dt, H, Nh, L, K, d_flags,
                                      stream);
    if (e == cudaSuccess) e = s4::launch_irfft_packed(K, H, L, stream);
    return cuda_status(e);
}

s4_status s4_fft_conv_workspace_size(int H, int L, size_t *bytes) {
    if (bytes == nullptr || H < 1) return S4_ERR_INVALID_ARG;
    if (!pow2_L(L)) return S4_ERR_UNSUPPORTED;
    *bytes = s4::conv_workspace_bytes(H, L);
    return S4_OK;
}

s4_status s4_fft_conv_prepare(const float *K, const float *D, int H, int L, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
    s4_status s = prepare_checks(K, D, H, L, workspace, workspace_bytes);
    if (s != S4_OK) return s;
    return cuda_status(s4::launch_kspec(K, D, H, L, workspace, stream));
}

s4_status s4_fft_conv_apply(const float *u, const void *workspace, int Bt, int H, int L, float *y,
                            size_t workspace_bytes, cudaStream_t stream) {
    s4_status s = conv_checks(u, Bt, H, L, y, workspace, workspace_bytes);
    if (s != S4_OK) return s;
    return cuda_status(s4::launch_fftconv(u, workspace, Bt, H, L, y, stream));
}

s4_status s4_fft_conv(const float *u, const float *K, const float *D, int Bt, int H, int L, float *y,
                      void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (D == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = conv_checks(u, Bt, H, L, y, workspace, workspace_bytes);
    if (s == S4_OK) s = prepare_checks(K, D, H, L, workspace, workspace_bytes);
    if (s != S4_OK) return s;
    const size_t nb = (size_t)Bt * H * L * sizeof(float);
    if (overlap(y, nb, K, (size_t)H * L * sizeof(float)) || overlap(y, nb, D, (size_t)H * sizeof(float)))
        return S4_ERR_INVALID_ARG;
    cudaError_t e = s4::launch_kspec(K, D, H, L, workspace, stream);
    if (e == cudaSuccess) e = s4::launch_fftconv(u, workspace, Bt, H, L, y, stream);
    return cuda_status(e);
}

s4_status s4_kernel_dplr_prepare(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                                 const s4_c32 *C, const float *log_dt, const float *D, int H, int Nh, int L,
                                 float *K, void *workspace, size_t workspace_bytes, unsigned *d_flags,
                                 cudaStream_t stream) {
    s4_status s = dplr_checks(Lambda, P, Q, B, C, log_dt, H, Nh, L, K);
    if (s == S4_OK) s = prepare_checks(K, D, H, L, workspace, workspace_bytes);
    if (s != S4_OK) return s;
    for (const void *p : {(const void *)Lambda, (const void *)P, (const void *)Q, (const void *)B,
                          (const void *)C})
        if (overlap(workspace, workspace_bytes, p, (size_t)H * Nh * sizeof(s4_c32))) return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_kgen((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q,
                                       (const float2 *)B, (const float2 *)C, log_dt, D, H, Nh, L, K, workspace,
                                       d_flags, stream));
}

s4_status s4_forward_dplr(const float *u, const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                          const s4_c32 *B, const s4_c32 *C, const float *log_dt, const float *D, int Bt, int H,
                          int Nh, int L, float *K, float *y, void *workspace, size_t workspace_bytes,
                          unsigned *d_flags, cudaStream_t stream) {
    if (D == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = conv_checks(u, Bt, H, L, y, workspace, workspace_bytes);
    if (s == S4_OK) s = dplr_checks(Lambda, P, Q, B, C, log_dt, H, Nh, L, K);
    if (s == S4_OK) s = prepare_checks(K, D, H, L, workspace, workspace_bytes);
    if (s != S4_OK) return s;
    const size_t nb = (size_t)Bt * H * L * sizeof(float), kb = (size_t)H * L * sizeof(float);
    if (overlap(y, nb, K, kb) || overlap(y, nb, D, (size_t)H * sizeof(float)) || overlap(u, nb, K, kb))
        return S4_ERR_INVALID_ARG;
    for (const void *p : {(const void *)Lambda, (const void *)P, (const void *)Q, (const void *)B,
                          (const void *)C})
        if (overlap(workspace, workspace_bytes, p, (size_t)H * Nh * sizeof(s4_c32)) ||
            overlap(y, nb, p, (size_t)H * Nh * sizeof(s4_c32)))
            return S4_ERR_INVALID_ARG;
    cudaError_t e = s4::launch_kgen((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q, (const float2 *)B,
                                    (const float2 *)C, log_dt, D, H, Nh, L, K, workspace, d_flags, stream);
    if (e == cudaSuccess) e = s4::launch_fftconv(u, workspace, Bt, H, L, y, stream);
    return cuda_status(e);
}

s4_status s4d_kernel_vandermonde(const s4_c32 *A, const s4_c32 *B, const s4_c32 *C, const float *log_dt,
                                 int H, int Nh, int L, float *K, unsigned *d_flags, cudaStream_t stream) {
    if (any_null(A, B, C) || log_dt == nullptr || K == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, L, true);
    if (s != S4_OK) return s;
    if (!params_aligned({A, B, C}) || !aligned(K, 16) || !aligned(log_dt, 4)) return S4_ERR_INVALID_ARG;
    const size_t kb = (size_t)H * L * sizeof(float), pb = (size_t)H * Nh * sizeof(s4_c32);
    if (overlap(K, kb, A, pb) || overlap(K, kb, B, pb) || overlap(K, kb, C, pb) ||
        overlap(K, kb, log_dt, (size_t)H * sizeof(float)))
        return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_vandermonde((const float2 *)A, (const float2 *)B, (const float2 *)C, log_dt,
                                              H, Nh, L, K, d_flags, stream));
}

s4_status s4_dplr_discretize(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                             const s4_c32 *C, const float *log_dt, int H, int Nh, s4_c32 *Abar,
                             s4_c32 *Bbar, s4_c32 *Cfull, cudaStream_t stream) {
    if (any_null(Lambda, P, Q, B, C) || any_null(Abar, Bbar, Cfull) || log_dt == nullptr)
        return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, 0, false);
    if (s != S4_OK) return s;
    if (!params_aligned({Lambda, P, Q, B, C, Abar, Bbar, Cfull})) return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_dplr_discretize((const float2 *)Lambda, (const float2 *)P,
                                                  (const float2 *)Q, (const float2 *)B, (const float2 *)C,
                                                  log_dt, H, Nh, (float2 *)Abar, (float2 *)Bbar,
                                                  (float2 *)Cfull, stream));
}

s4_status s4_dplr_discretize_structured(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                                        const s4_c32 *B, const float *log_dt, int H, int Nh, s4_c32 *Astr,
                                        s4_c32 *Bbar, cudaStream_t stream) {
    if (any_null(Lambda, P, Q, B) || any_null(Astr, Bbar) || log_dt == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, 0, false);
    if (s != S4_OK) return s;
    if (!params_aligned({Lambda, P, Q, B, Astr, Bbar})) return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_dplr_discretize_structured((const float2 *)Lambda, (const float2 *)P,
                                                             (const float2 *)Q, (const float2 *)B, log_dt, H,
                                                             Nh, (float2 *)Astr, (float2 *)Bbar, stream));
}

s4_status s4d_discretize_zoh(const s4_c32 *A, const s4_c32 *B, const float *log_dt, int H, int Nh,
                             s4_c32 *Abar, s4_c32 *Bbar, cudaStream_t stream) {
    if (any_null(A, B) || any_null(Abar, Bbar) || log_dt == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, 0, false);
    if (s != S4_OK) return s;
    if (!params_aligned({A, B, Abar, Bbar})) return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_s4d_zoh((const float2 *)A, (const float2 *)B, log_dt, H, Nh,
                                          (float2 *)Abar, (float2 *)Bbar, stream));
}

static s4_status step_checks(s4_step_mode mode, const s4_c32 *Abar, const s4_c32 *Bbar, const s4_c32 *C,
                             const float *D, int Bt, int H, int Ns, int T, const s4_c32 *x, const float *u,
                             const float *y) {
    if (any_null(Abar, Bbar, C, x) || any_null(D, u, y)) return S4_ERR_INVALID_ARG;
    if (Bt < 1 || H < 1 || Ns < 1 || T < 1) return S4_ERR_INVALID_ARG;
    if (H > S4_MAX_H) return S4_ERR_UNSUPPORTED;
    if (mode == S4_STEP_DENSE) {
        if (Ns > S4_MAX_DENSE_N) return S4_ERR_UNSUPPORTED;
    } else if (mode == S4_STEP_DIAG || mode == S4_STEP_DPLR) {
        if (Ns > S4_MAX_NH) return S4_ERR_UNSUPPORTED;
    } else {
        return S4_ERR_INVALID_ARG;
    }
    if (!params_aligned({Abar, Bbar, C, x})) return S4_ERR_INVALID_ARG;
    const size_t xb = (size_t)Bt * H * Ns * sizeof(s4_c32), yb = (size_t)Bt * H * T * sizeof(float);
    if (overlap(x, xb, y, yb) || overlap(u, yb, y, yb)) return S4_ERR_INVALID_ARG;
    return S4_OK;
}

s4_status s4_recurrent_step(s4_step_mode mode, const s4_c32 *Abar, const s4_c32 *Bbar, const s4_c32 *C,
                            const float *D, int Bt, int H, int Ns, s4_c32 *x, const float *u_t, float *y_t,
                            cudaStream_t stream) {
    s4_status s = step_checks(mode, Abar, Bbar, C, D, Bt, H, Ns, 1, x, u_t, y_t);
    if (s != S4_OK) return s;
    return cuda_status(s4::launch_step((int)mode, (const float2 *)Abar, (const float2 *)Bbar, (const float2 *)C,
                                       D, Bt, H, Ns, 1, (float2 *)x, u_t, y_t, stream));
}

s4_status s4_recurrent_scan(s4_step_mode mode, const s4_c32 *Abar, const s4_c32 *Bbar, const s4_c32 *C,
                            const float *D, int Bt, int H, int Ns, int T, s4_c32 *x, const float *u, float *y,
                            cudaStream_t stream) {
    s4_status s = step_checks(mode, Abar, Bbar, C, D, Bt, H, Ns, T, x, u, y);
    if (s != S4_OK) return s;
    return cuda_status(s4::launch_step((int)mode, (const float2 *)Abar, (const float2 *)Bbar, (const float2 *)C,
                                       D, Bt, H, Ns, T, (float2 *)x, u, y, stream));
}

}  // extern "C"
