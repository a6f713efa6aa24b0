// api.cu -- the extern "C" entry points of libs4dplr.so (declared and
// documented in include/s4dplr.h). Every argument is checked on the host
// before anything is launched; nothing here allocates device memory.
#include <cstdint>
#include <vector>

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

// Ordering events of the host-buffer pipeline, created once per (host
// thread, device) and reused by every later call: an event may be recorded
// again as soon as the waits on its previous record are enqueued, which the
// pipeline does in order. They live until the process exits.
cudaError_t pipeline_events(size_t n, cudaEvent_t **out) {
    thread_local std::vector<cudaEvent_t> pools[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::vector<cudaEvent_t> &pool = pools[dev & 63];
    while (pool.size() < n) {
        cudaEvent_t ev = nullptr;
        e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        pool.push_back(ev);
    }
    *out = pool.data();
    return cudaSuccess;
}

// The same pipeline when the batch has fewer row pairs than chunks asked for
// (L <= 16384, where the workspace is only the per-channel spectrum, so the
// spectrum of channels [h0, h1) starts at h0 * 2L complex values): each row
// pair is also cut into channel slices. Chunk (pair, slice) is staged in
// u_dev / y_dev as a contiguous [rows][h1 - h0][L] block at
// b0 H L + rows h0 L (one copy per row each way) and convolved as a batch of
// its own; the blocks tile the buffers without overlap.
cudaError_t conv_host_pipeline_sliced(const float *u_host, const void *ws, int Bt, int H, int L, float *y_host,
                                      float *u_dev, float *y_dev, int nchunks, cudaStream_t st, cudaStream_t h2d,
                                      cudaStream_t d2h, cudaEvent_t start) {
    const int npairs = (Bt + 1) / 2;
    int slices = (nchunks + npairs - 1) / npairs;
    if (slices > H) slices = H;
    const int hc = (H + slices - 1) / slices;
    slices = (H + hc - 1) / hc;
    const int total = npairs * slices;
    cudaEvent_t *ev = nullptr;   // [2 total + 1]: upload c done, convolution c done, last download done
    cudaError_t e = pipeline_events(2 * (size_t)total + 1, &ev);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h2d, start, 0);
    for (int c = 0; c < total && e == cudaSuccess; ++c) {
        const int pr = c / slices, q = c % slices;
        const int b0 = 2 * pr, nb = b0 + 1 < Bt ? 2 : 1;
        const int h0 = q * hc, nh = h0 + hc < H ? hc : H - h0;
        const size_t blk = (size_t)b0 * H * L + (size_t)nb * h0 * L, rowb = (size_t)nh * L;
        for (int r = 0; r < nb && e == cudaSuccess; ++r)
            e = cudaMemcpyAsync(u_dev + blk + r * rowb, u_host + ((size_t)(b0 + r) * H + h0) * L,
                                rowb * sizeof(float), cudaMemcpyHostToDevice, h2d);
        if (e == cudaSuccess) e = cudaEventRecord(ev[2 * c], h2d);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev[2 * c], 0);
        if (e == cudaSuccess)
            e = s4::launch_fftconv(u_dev + blk, (const char *)ws + (size_t)h0 * 2 * L * 2 * sizeof(float), nb, nh, L,
                                   y_dev + blk, st);
        if (e == cudaSuccess) e = cudaEventRecord(ev[2 * c + 1], st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(d2h, ev[2 * c + 1], 0);
        for (int r = 0; r < nb && e == cudaSuccess; ++r)
            e = cudaMemcpyAsync(y_host + ((size_t)(b0 + r) * H + h0) * L, y_dev + blk + r * rowb,
                                rowb * sizeof(float), cudaMemcpyDeviceToHost, d2h);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev[2 * total], d2h);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev[2 * total], 0);
    return e;
}

// The convolution of a batch held in host memory. Chunk c (whole row pairs)
// is uploaded on h2d, convolved on st once it has arrived and downloaded on
// d2h once convolved, so uploads, convolutions and downloads of consecutive
// chunks overlap (the two copy directions use separate copy engines). The
// uploads start only after the work already queued on st (an earlier call
// may still read u_dev or write y_dev); st waits for the last download, so a
// caller that synchronises st sees y_host complete.
cudaError_t conv_host_pipeline(const float *u_host, const void *ws, int Bt, int H, int L, float *y_host,
                               float *u_dev, float *y_dev, int nchunks, cudaStream_t st, cudaStream_t h2d,
                               cudaStream_t d2h, cudaEvent_t start) {
    const int npairs = (Bt + 1) / 2;
    if (nchunks > npairs && H > 1 && L <= 16384)
        return conv_host_pipeline_sliced(u_host, ws, Bt, H, L, y_host, u_dev, y_dev, nchunks, st, h2d, d2h, start);
    if (nchunks > npairs) nchunks = npairs;
    const int pairs_per_chunk = (npairs + nchunks - 1) / nchunks;
    nchunks = (npairs + pairs_per_chunk - 1) / pairs_per_chunk;
    const size_t row = (size_t)H * L;
    cudaEvent_t *ev = nullptr;   // [2 nchunks + 1]: upload c done, convolution c done, last download done
    cudaError_t e = pipeline_events(2 * (size_t)nchunks + 1, &ev);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h2d, start, 0);
    for (int c = 0; c < nchunks && e == cudaSuccess; ++c) {
        const int b0 = 2 * c * pairs_per_chunk;
        const int b1 = (b0 + 2 * pairs_per_chunk) < Bt ? b0 + 2 * pairs_per_chunk : Bt;
        const size_t off = (size_t)b0 * row, bytes = (size_t)(b1 - b0) * row * sizeof(float);
        e = cudaMemcpyAsync(u_dev + off, u_host + off, bytes, cudaMemcpyHostToDevice, h2d);
        if (e == cudaSuccess) e = cudaEventRecord(ev[2 * c], h2d);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev[2 * c], 0);
        if (e == cudaSuccess) e = s4::launch_fftconv(u_dev + off, ws, b1 - b0, H, L, y_dev + off, st);
        if (e == cudaSuccess) e = cudaEventRecord(ev[2 * c + 1], st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(d2h, ev[2 * c + 1], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(y_host + off, y_dev + off, bytes, cudaMemcpyDeviceToHost, d2h);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev[2 * nchunks], d2h);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev[2 * nchunks], 0);
    return e;
}

// checks shared by the two host-buffer entry points
s4_status host_buffer_checks(const float *u_host, const float *y_host, const float *u_dev, const float *y_dev,
                             int Bt, int H, int L, const void *ws, size_t ws_bytes, int nchunks) {
    if (any_null(u_host, y_host) || nchunks < 1) return S4_ERR_INVALID_ARG;
    s4_status s = conv_checks(u_dev, Bt, H, L, y_dev, ws, ws_bytes);
    if (s != S4_OK) return s;
    const size_t nb = (size_t)Bt * H * L * sizeof(float);
    if (overlap(u_host, nb, y_host, nb) || overlap(u_dev, nb, ws, ws_bytes)) return S4_ERR_INVALID_ARG;
    return S4_OK;
}

// [Bt, H, L] activations of the S4Block entry points
s4_status block_shape_checks(int Bt, int H, int L) {
    if (Bt < 1 || H < 1 || H > S4_MAX_BLOCK_H) return S4_ERR_INVALID_ARG;
    if (!pow2_L(L)) return S4_ERR_UNSUPPORTED;
    if ((double)Bt * (double)H * (double)L >= 1099511627776.0) return S4_ERR_INVALID_ARG;   // 2^40
    return S4_OK;
}

s4_status layernorm_checks(const float *x, const float *gamma, const float *beta, float eps, int Bt, int H, int L,
                           const float *z) {
    if (any_null(x, gamma, beta, z)) return S4_ERR_INVALID_ARG;
    s4_status s = block_shape_checks(Bt, H, L);
    if (s != S4_OK) return s;
    if (!(eps > 0.0f) || !(eps < 3.0e38f)) return S4_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(z, 16) || !aligned(gamma, 4) || !aligned(beta, 4)) return S4_ERR_INVALID_ARG;
    const size_t nb = (size_t)Bt * H * L * sizeof(float);
    if (z != x && overlap(x, nb, z, nb)) return S4_ERR_INVALID_ARG;
    if (overlap(z, nb, gamma, (size_t)H * 4) || overlap(z, nb, beta, (size_t)H * 4)) return S4_ERR_INVALID_ARG;
    return S4_OK;
}

s4_status glu_checks(const float *y, const float *x, const float *bias, const void *ws, size_t ws_bytes, int Bt,
                     int H, int L, const float *out) {
    if (any_null(y, x, bias, out) || ws == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = block_shape_checks(Bt, H, L);
    if (s != S4_OK) return s;
    if (!aligned(y, 16) || !aligned(x, 16) || !aligned(out, 16) || !aligned(bias, 4)) return S4_ERR_INVALID_ARG;
    if (!aligned(ws, 256) || ws_bytes < s4::glu_workspace_bytes(H)) return S4_ERR_WORKSPACE;
    const size_t nb = (size_t)Bt * H * L * sizeof(float);
    if (overlap(out, nb, y, nb) || overlap(out, nb, ws, ws_bytes) || overlap(out, nb, bias, (size_t)2 * H * 4))
        return S4_ERR_INVALID_ARG;
    if (out != x && overlap(out, nb, x, nb)) return S4_ERR_INVALID_ARG;
    return S4_OK;
}

// an event marking the work queued on st so far (the pipeline's own events
// follow it in the pool, so it is recorded before they are)
cudaError_t mark(cudaStream_t st, cudaEvent_t *ev) {
    thread_local cudaEvent_t marks[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaEvent_t &m = marks[dev & 63];
    if (m == nullptr) e = cudaEventCreateWithFlags(&m, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventRecord(m, st);
    *ev = m;
    return e;
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

s4_status s4_fft_conv_apply_adjoint(const float *dy, const void *workspace, int Bt, int H, int L, float *du,
                                    size_t workspace_bytes, cudaStream_t stream) {
    s4_status s = conv_checks(dy, Bt, H, L, du, workspace, workspace_bytes);
    if (s != S4_OK) return s;
    return cuda_status(s4::launch_fftconv(dy, workspace, Bt, H, L, du, stream, true));
}

s4_status s4_fft_conv_kernel_grad_workspace_size(int H, int L, size_t *bytes) {
    if (bytes == nullptr || H < 1) return S4_ERR_INVALID_ARG;
    if (!pow2_L(L)) return S4_ERR_UNSUPPORTED;
    *bytes = s4::corr_workspace_bytes(H, L);
    return S4_OK;
}

s4_status s4_fft_conv_kernel_grad(const float *u, const float *dy, int Bt, int H, int L, float *dK, float *dD,
                                  void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (any_null(u, dy, dK) || workspace == nullptr) return S4_ERR_INVALID_ARG;
    if (Bt < 1 || H < 1) return S4_ERR_INVALID_ARG;
    if (!pow2_L(L)) return S4_ERR_UNSUPPORTED;
    if ((double)Bt * (double)H * (double)L >= 1099511627776.0) return S4_ERR_INVALID_ARG;   // 2^40
    if (!aligned(u, 16) || !aligned(dy, 16) || !aligned(dK, 16) || (dD != nullptr && !aligned(dD, 4)))
        return S4_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || workspace_bytes < s4::corr_workspace_bytes(H, L)) return S4_ERR_WORKSPACE;
    const size_t nb = (size_t)Bt * H * L * sizeof(float), kb = (size_t)H * L * sizeof(float);
    const size_t hb = (size_t)H * sizeof(float);
    for (const void *p : {(const void *)u, (const void *)dy}) {
        if (overlap(p, nb, dK, kb) || overlap(p, nb, workspace, workspace_bytes)) return S4_ERR_INVALID_ARG;
        if (dD != nullptr && overlap(p, nb, dD, hb)) return S4_ERR_INVALID_ARG;
    }
    if (overlap(dK, kb, workspace, workspace_bytes)) return S4_ERR_INVALID_ARG;
    if (dD != nullptr && (overlap(dD, hb, dK, kb) || overlap(dD, hb, workspace, workspace_bytes)))
        return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_corr(u, dy, Bt, H, L, dK, dD, workspace, stream));
}

namespace {
s4_status kbwd_checks(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B, const s4_c32 *C,
                      const float *log_dt, const float *dK, int H, int Nh, int L, s4_c32 *dLambda, s4_c32 *dP,
                      s4_c32 *dQ, s4_c32 *dB, s4_c32 *dC, float *dlog_dt) {
    if (any_null(Lambda, P, Q, B, C) || any_null(dLambda, dP, dQ, dB, dC) || any_null(log_dt, dK, dlog_dt))
        return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, L, true);
    if (s != S4_OK) return s;
    if (!params_aligned({Lambda, P, Q, B, C, dLambda, dP, dQ, dB, dC}) || !aligned(dK, 4)) return S4_ERR_INVALID_ARG;
    const size_t pb = (size_t)H * Nh * sizeof(s4_c32);
    const void *outs[] = {dLambda, dP, dQ, dB, dC};
    const void *ins[] = {Lambda, P, Q, B, C};
    for (int i = 0; i < 5; ++i) {
        for (int j = 0; j < 5; ++j) {
            if (overlap(outs[i], pb, ins[j], pb)) return S4_ERR_INVALID_ARG;
            if (j > i && overlap(outs[i], pb, outs[j], pb)) return S4_ERR_INVALID_ARG;
        }
        if (overlap(outs[i], pb, dK, (size_t)H * L * sizeof(float)) ||
            overlap(outs[i], pb, dlog_dt, (size_t)H * sizeof(float)))
            return S4_ERR_INVALID_ARG;
    }
    return S4_OK;
}
}  // namespace

s4_status s4_kernel_dplr_backward(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                                  const s4_c32 *C, const float *log_dt, const float *dK, int H, int Nh, int L,
                                  s4_c32 *dLambda, s4_c32 *dP, s4_c32 *dQ, s4_c32 *dB, s4_c32 *dC,
                                  float *dlog_dt, cudaStream_t stream) {
    s4_status s = kbwd_checks(Lambda, P, Q, B, C, log_dt, dK, H, Nh, L, dLambda, dP, dQ, dB, dC, dlog_dt);
    if (s != S4_OK) return s;
    if (L > 16384) return S4_ERR_UNSUPPORTED;   // needs the workspace form
    return cuda_status(s4::launch_kgen_backward((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q,
                                                (const float2 *)B, (const float2 *)C, log_dt, dK, H, Nh, L,
                                                (float2 *)dLambda, (float2 *)dP, (float2 *)dQ, (float2 *)dB,
                                                (float2 *)dC, dlog_dt, nullptr, stream));
}

s4_status s4_kernel_dplr_backward_workspace_size(int H, int L, size_t *bytes) {
    if (bytes == nullptr || H < 1) return S4_ERR_INVALID_ARG;
    if (!pow2_L(L)) return S4_ERR_UNSUPPORTED;
    *bytes = s4::kgen_backward_workspace_bytes(H, L);
    return S4_OK;
}

s4_status s4_kernel_dplr_backward_ws(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                                     const s4_c32 *C, const float *log_dt, const float *dK, int H, int Nh, int L,
                                     s4_c32 *dLambda, s4_c32 *dP, s4_c32 *dQ, s4_c32 *dB, s4_c32 *dC,
                                     float *dlog_dt, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    s4_status s = kbwd_checks(Lambda, P, Q, B, C, log_dt, dK, H, Nh, L, dLambda, dP, dQ, dB, dC, dlog_dt);
    if (s != S4_OK) return s;
    const size_t need = s4::kgen_backward_workspace_bytes(H, L);
    if (need > 0) {
        if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need) return S4_ERR_WORKSPACE;
        const size_t pb = (size_t)H * Nh * sizeof(s4_c32);
        for (const void *o : {(const void *)dLambda, (const void *)dP, (const void *)dQ, (const void *)dB,
                              (const void *)dC, (const void *)dlog_dt, (const void *)dK})
            if (overlap(o, o == dK ? (size_t)H * L * sizeof(float) : pb, workspace, workspace_bytes))
                return S4_ERR_INVALID_ARG;
    }
    return cuda_status(s4::launch_kgen_backward((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q,
                                                (const float2 *)B, (const float2 *)C, log_dt, dK, H, Nh, L,
                                                (float2 *)dLambda, (float2 *)dP, (float2 *)dQ, (float2 *)dB,
                                                (float2 *)dC, dlog_dt, need > 0 ? workspace : nullptr, stream));
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

s4_status s4_fft_conv_host(const float *u_host, const float *K, const float *D, int Bt, int H, int L,
                           float *y_host, float *u_dev, float *y_dev, void *workspace, size_t workspace_bytes,
                           int nchunks, cudaStream_t stream, cudaStream_t h2d_stream, cudaStream_t d2h_stream) {
    if (D == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = host_buffer_checks(u_host, y_host, u_dev, y_dev, Bt, H, L, workspace, workspace_bytes, nchunks);
    if (s == S4_OK) s = prepare_checks(K, D, H, L, workspace, workspace_bytes);
    if (s != S4_OK) return s;
    const size_t nb = (size_t)Bt * H * L * sizeof(float), kb = (size_t)H * L * sizeof(float);
    if (overlap(y_dev, nb, K, kb) || overlap(u_dev, nb, K, kb) || overlap(y_dev, nb, D, (size_t)H * sizeof(float)))
        return S4_ERR_INVALID_ARG;
    cudaEvent_t start = nullptr;
    cudaError_t e = mark(stream, &start);
    if (e == cudaSuccess) e = s4::launch_kspec(K, D, H, L, workspace, stream);
    if (e == cudaSuccess)
        e = conv_host_pipeline(u_host, workspace, Bt, H, L, y_host, u_dev, y_dev, nchunks, stream, h2d_stream,
                               d2h_stream, start);
    return cuda_status(e);
}

s4_status s4_forward_dplr_host(const float *u_host, const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q,
                               const s4_c32 *B, const s4_c32 *C, const float *log_dt, const float *D, int Bt,
                               int H, int Nh, int L, float *y_host, float *K, float *u_dev, float *y_dev,
                               void *workspace, size_t workspace_bytes, unsigned *d_flags, int nchunks,
                               cudaStream_t stream, cudaStream_t h2d_stream, cudaStream_t d2h_stream) {
    if (D == nullptr) return S4_ERR_INVALID_ARG;
    s4_status s = host_buffer_checks(u_host, y_host, u_dev, y_dev, Bt, H, L, workspace, workspace_bytes, nchunks);
    if (s == S4_OK) s = dplr_checks(Lambda, P, Q, B, C, log_dt, H, Nh, L, K);
    if (s == S4_OK) s = prepare_checks(K, D, H, L, workspace, workspace_bytes);
    if (s != S4_OK) return s;
    const size_t nb = (size_t)Bt * H * L * sizeof(float), kb = (size_t)H * L * sizeof(float);
    if (overlap(y_dev, nb, K, kb) || overlap(u_dev, nb, K, kb) || overlap(y_dev, nb, D, (size_t)H * sizeof(float)))
        return S4_ERR_INVALID_ARG;
    for (const void *p : {(const void *)Lambda, (const void *)P, (const void *)Q, (const void *)B,
                          (const void *)C})
        if (overlap(workspace, workspace_bytes, p, (size_t)H * Nh * sizeof(s4_c32)) ||
            overlap(y_dev, nb, p, (size_t)H * Nh * sizeof(s4_c32)) ||
            overlap(u_dev, nb, p, (size_t)H * Nh * sizeof(s4_c32)))
            return S4_ERR_INVALID_ARG;
    cudaEvent_t start = nullptr;
    cudaError_t e = mark(stream, &start);   // the first upload overlaps the kernel generation
    if (e == cudaSuccess)
        e = s4::launch_kgen((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q, (const float2 *)B,
                            (const float2 *)C, log_dt, D, H, Nh, L, K, workspace, d_flags, stream);
    if (e == cudaSuccess)
        e = conv_host_pipeline(u_host, workspace, Bt, H, L, y_host, u_dev, y_dev, nchunks, stream, h2d_stream,
                               d2h_stream, start);
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

s4_status s4_dplr_ctilde(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *C,
                         const float *log_dt, int H, int Nh, int L, s4_c32 *Ctilde, cudaStream_t stream) {
    if (any_null(Lambda, P, Q, C) || Ctilde == nullptr || log_dt == nullptr) return S4_ERR_INVALID_ARG;
    if (L < 1) return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, 0, false);
    if (s != S4_OK) return s;
    if (!params_aligned({Lambda, P, Q, C, Ctilde})) return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_dplr_ctilde((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q,
                                              (const float2 *)C, log_dt, H, Nh, L, (float2 *)Ctilde, stream));
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

// ---------------------------------------------------------------- S4Block
s4_status s4_layernorm_channels(const float *x, const float *gamma, const float *beta, float eps, int Bt, int H,
                                int L, float *z, cudaStream_t stream) {
    s4_status s = layernorm_checks(x, gamma, beta, eps, Bt, H, L, z);
    if (s != S4_OK) return s;
    return cuda_status(s4::launch_layernorm_channels(x, gamma, beta, eps, Bt, H, L, z, stream));
}

s4_status s4_glu_projection_workspace_size(int H, size_t *bytes) {
    if (bytes == nullptr || H < 1 || H > S4_MAX_BLOCK_H) return S4_ERR_INVALID_ARG;
    *bytes = s4::glu_workspace_bytes(H);
    return S4_OK;
}

s4_status s4_glu_projection_prepare(const float *W, int H, void *workspace, size_t workspace_bytes,
                                    cudaStream_t stream) {
    if (W == nullptr || workspace == nullptr || H < 1 || H > S4_MAX_BLOCK_H) return S4_ERR_INVALID_ARG;
    if (!aligned(W, 4)) return S4_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || workspace_bytes < s4::glu_workspace_bytes(H)) return S4_ERR_WORKSPACE;
    if (overlap(W, (size_t)2 * H * H * sizeof(float), workspace, workspace_bytes)) return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_glu_prepare(W, H, workspace, stream));
}

s4_status s4_glu_projection_residual(const float *y, const float *x, const float *bias, const void *workspace,
                                     size_t workspace_bytes, int Bt, int H, int L, float *out, unsigned *d_flags,
                                     cudaStream_t stream) {
    s4_status s = glu_checks(y, x, bias, workspace, workspace_bytes, Bt, H, L, out);
    if (s != S4_OK) return s;
    return cuda_status(s4::launch_glu_projection(y, x, bias, workspace, Bt, H, L, out, d_flags, stream));
}

s4_status s4_block_forward(const float *x, const float *gamma, const float *beta, float eps,
                           const void *conv_workspace, size_t conv_workspace_bytes, const float *bias,
                           const void *glu_workspace, size_t glu_workspace_bytes, int Bt, int H, int L, float *z,
                           float *y, float *out, unsigned *d_flags, cudaStream_t stream) {
    s4_status s = layernorm_checks(x, gamma, beta, eps, Bt, H, L, z);
    if (s == S4_OK && z == x) s = S4_ERR_INVALID_ARG;   // x is still needed for the residual
    if (s == S4_OK) s = conv_checks(z, Bt, H, L, y, conv_workspace, conv_workspace_bytes);
    if (s == S4_OK) s = glu_checks(y, x, bias, glu_workspace, glu_workspace_bytes, Bt, H, L, out);
    if (s != S4_OK) return s;
    const size_t nb = (size_t)Bt * H * L * sizeof(float);
    if (overlap(x, nb, y, nb) || overlap(z, nb, out, nb) || overlap(z, nb, glu_workspace, glu_workspace_bytes) ||
        overlap(y, nb, glu_workspace, glu_workspace_bytes) || overlap(z, nb, conv_workspace, conv_workspace_bytes) ||
        overlap(out, nb, conv_workspace, conv_workspace_bytes))
        return S4_ERR_INVALID_ARG;
    cudaError_t e = s4::launch_layernorm_channels(x, gamma, beta, eps, Bt, H, L, z, stream);
    if (e == cudaSuccess) e = s4::launch_fftconv(z, conv_workspace, Bt, H, L, y, stream);
    if (e == cudaSuccess) e = s4::launch_glu_projection(y, x, bias, glu_workspace, Bt, H, L, out, d_flags, stream);
    return cuda_status(e);
}

// ------------------------------------------------------- ZOH of the DPLR system
s4_status s4_dplr_discretize_zoh(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                                 const s4_c32 *C, const float *log_dt, int H, int Nh, s4_c32 *Abar, s4_c32 *Bbar,
                                 s4_c32 *Cfull, cudaStream_t stream) {
    if (any_null(Lambda, P, Q, B, C) || any_null(Abar, Bbar, Cfull) || log_dt == nullptr)
        return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, 0, false);
    if (s != S4_OK) return s;
    if (Nh > S4_MAX_ZOH_NH) return S4_ERR_UNSUPPORTED;
    if (!params_aligned({Lambda, P, Q, B, C, Abar, Bbar, Cfull}) || !aligned(log_dt, 4)) return S4_ERR_INVALID_ARG;
    const size_t N = 2 * (size_t)Nh, ab = (size_t)H * N * N * sizeof(s4_c32), vb = (size_t)H * N * sizeof(s4_c32);
    if (overlap(Abar, ab, Bbar, vb) || overlap(Abar, ab, Cfull, vb) || overlap(Bbar, vb, Cfull, vb))
        return S4_ERR_INVALID_ARG;
    return cuda_status(s4::launch_dplr_zoh((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q,
                                           (const float2 *)B, (const float2 *)C, log_dt, H, Nh, 0, (float2 *)Abar,
                                           (float2 *)Bbar, (float2 *)Cfull, nullptr, nullptr, stream));
}

s4_status s4_kernel_dplr_zoh(const s4_c32 *Lambda, const s4_c32 *P, const s4_c32 *Q, const s4_c32 *B,
                             const s4_c32 *C, const float *log_dt, int H, int Nh, int L, float *K,
                             unsigned *d_flags, cudaStream_t stream) {
    s4_status s = dplr_checks(Lambda, P, Q, B, C, log_dt, H, Nh, L, K);
    if (s != S4_OK) return s;
    if (Nh > S4_MAX_ZOH_NH) return S4_ERR_UNSUPPORTED;
    return cuda_status(s4::launch_dplr_zoh((const float2 *)Lambda, (const float2 *)P, (const float2 *)Q,
                                           (const float2 *)B, (const float2 *)C, log_dt, H, Nh, L, nullptr, nullptr,
                                           nullptr, K, d_flags, stream));
}

// ----------------------------------------------------------- S4D backward
s4_status s4d_kernel_vandermonde_backward(const s4_c32 *A, const s4_c32 *B, const s4_c32 *C, const float *log_dt,
                                          const float *dK, int H, int Nh, int L, s4_c32 *dA, s4_c32 *dB,
                                          s4_c32 *dC, float *dlog_dt, cudaStream_t stream) {
    if (any_null(A, B, C) || any_null(dA, dB, dC) || any_null(log_dt, dK, dlog_dt)) return S4_ERR_INVALID_ARG;
    s4_status s = check_modes(H, Nh, L, true);
    if (s != S4_OK) return s;
    if (!params_aligned({A, B, C, dA, dB, dC}) || !aligned(dK, 4) || !aligned(log_dt, 4) || !aligned(dlog_dt, 4))
        return S4_ERR_INVALID_ARG;
    const size_t pb = (size_t)H * Nh * sizeof(s4_c32);
    const void *outs[] = {dA, dB, dC};
    const void *ins[] = {A, B, C};
    for (int i = 0; i < 3; ++i) {
        for (int k = 0; k < 3; ++k) {
            if (overlap(outs[i], pb, ins[k], pb)) return S4_ERR_INVALID_ARG;
            if (k > i && overlap(outs[i], pb, outs[k], pb)) return S4_ERR_INVALID_ARG;
        }
        if (overlap(outs[i], pb, dK, (size_t)H * L * sizeof(float)) ||
            overlap(outs[i], pb, dlog_dt, (size_t)H * sizeof(float)))
            return S4_ERR_INVALID_ARG;
    }
    return cuda_status(s4::launch_vandermonde_backward((const float2 *)A, (const float2 *)B, (const float2 *)C,
                                                       log_dt, dK, H, Nh, L, (float2 *)dA, (float2 *)dB,
                                                       (float2 *)dC, dlog_dt, stream));
}

}  // extern "C"
