// noalloc.cu -- s4_fft_conv_static: the FFT convolution of s4_fft_conv with
// its workspace in a fixed device array owned by the library, for callers
// that cannot allocate device memory themselves (a plugin inside a host
// application whose memory pool owns the GPU, or a real-time path where the
// implicit device synchronisation of cudaMalloc is not allowed).
//
// The scratch is one file-scope __device__ array of S4_STATIC_SCRATCH_BYTES.
// Host code must not use the array's name as a device address (on the host
// it is only a stand-in symbol), so its device address is fetched once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call made on that device, and passed to the kernels.
#include <mutex>

#include "launch.h"
#include "s4dplr.h"

namespace {

static __device__ __align__(256) unsigned char g_conv_scratch[S4_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct DeviceScratch {
    std::once_flag once;
    void *ptr = nullptr;
    cudaError_t err = cudaSuccess;
};
DeviceScratch g_scratch[kMaxDevices];

cudaError_t scratch_of_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    DeviceScratch &d = g_scratch[dev];
    std::call_once(d.once, [&d] { d.err = cudaGetSymbolAddress(&d.ptr, g_conv_scratch); });
    if (d.err != cudaSuccess) return d.err;
    *out = d.ptr;
    return cudaSuccess;
}

bool is_aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Buffers of another device, or unregistered host memory, would be illegal
// addresses for the kernels on the current device (whose scratch is used).
bool on_current_device(const void *p, int dev) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();   // a failed query leaves its error behind: clear it
        return false;
    }
    if (a.type == cudaMemoryTypeUnregistered) return false;
    return a.type != cudaMemoryTypeDevice || a.device == dev;
}

bool ranges_overlap(const void *a, size_t an, const void *b, size_t bn) {
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + bn && y < x + an;
}

}  // namespace

extern "C" s4_status s4_fft_conv_static(const float *u, const float *K, const float *D, int Bt, int H,
                                        int L, float *y, cudaStream_t stream) {
    if (u == nullptr || K == nullptr || D == nullptr || y == nullptr) return S4_ERR_INVALID_ARG;
    if (Bt < 1 || H < 1) return S4_ERR_INVALID_ARG;
    if (L < S4_MIN_L || L > S4_MAX_L || (L & (L - 1)) != 0) return S4_ERR_UNSUPPORTED;
    if ((double)Bt * (double)H * (double)L >= 1099511627776.0) return S4_ERR_INVALID_ARG;   // 2^40
    if (!is_aligned(u, 16) || !is_aligned(y, 16) || !is_aligned(K, 16) || !is_aligned(D, 4))
        return S4_ERR_INVALID_ARG;
    const size_t nb = (size_t)Bt * H * L * sizeof(float), kb = (size_t)H * L * sizeof(float);
    if (ranges_overlap(u, nb, y, nb) || ranges_overlap(y, nb, K, kb) ||
        ranges_overlap(y, nb, D, (size_t)H * sizeof(float)))
        return S4_ERR_INVALID_ARG;
    if (s4::conv_workspace_bytes(H, L) > (size_t)S4_STATIC_SCRATCH_BYTES) return S4_ERR_UNSUPPORTED;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        s4::record_cuda_error(e);
        return S4_ERR_CUDA;
    }
    if (!on_current_device(u, dev) || !on_current_device(K, dev) || !on_current_device(D, dev) ||
        !on_current_device(y, dev))
        return S4_ERR_INVALID_ARG;
    void *ws = nullptr;
    e = scratch_of_current_device(&ws);
    if (e == cudaSuccess) e = s4::launch_kspec(K, D, H, L, ws, stream);
    if (e == cudaSuccess) e = s4::launch_fftconv(u, ws, Bt, H, L, y, stream);
    if (e != cudaSuccess) {
        s4::record_cuda_error(e);
        return S4_ERR_CUDA;
    }
    return S4_OK;
}
