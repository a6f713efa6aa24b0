// kgen.cu -- the DPLR kernel K and the spectrum of the zero-padded K + D
// delta_0 in one launch ("The S4 kernel, from scratch", §4 and §5), for
// L <= 8192. One CTA per channel:
//   A. the Cauchy/Woodbury generating function at j = 0 .. L/2 (cauchy.cuh),
//      written with its conjugate mirror straight into the digit-reversed
//      positions the inverse transform reads;
//   B. length-L inverse transform (decimation in time) -> K, stored;
//   C. the same registers start the length-2L forward transform of the
//      zero-padded K (both halves of the transform, as in k_fftconv_pair);
//      its spectrum, plus D and times 1/2L, goes to the convolution workspace
//      in the layout k_fftconv_pair reads.
// Longer kernels take k_cauchy, then (L = 16384) the inverse transform fused
// with the spectrum in k_kspec_quad_pair, or (L >= 32768) k_irfft + k_kspec.
#include "launch.h"
#include "pairs.cuh"

namespace s4 {

template <int LG>
__global__ void __launch_bounds__(pair_threads<LG>(), pair_min_blocks<LG>())
k_kgen(const float2 *__restrict__ Lambda, const float2 *__restrict__ P, const float2 *__restrict__ Q,
       const float2 *__restrict__ B, const float2 *__restrict__ Cc, const float *__restrict__ log_dt,
       const float *__restrict__ D, int Nh, float *__restrict__ K, float2 *__restrict__ spec,
       unsigned *__restrict__ flags) {
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    pair_tables<LG>(s);
    const int h = blockIdx.x;
    kgen_channel<LG>(s, Lambda, P, Q, B, Cc, log_dt, D, Nh, h, K, spec + (size_t)h * 2 * (1 << LG), flags);
}

namespace {
template <int LG>
cudaError_t run_kgen(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B, const float2 *C,
                     const float *log_dt, const float *D, int H, int Nh, float *K, void *ws, unsigned *flags,
                     cudaStream_t st) {
    constexpr int T = pair_threads<LG>();
    const size_t smem = pair_smem_bytes<LG>(Nh);
    static int configured_smem[64];   // per device: largest opt-in done so far
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (smem > 48 * 1024 && configured_smem[dev & 63] < (int)smem) {
        e = cudaFuncSetAttribute(k_kgen<LG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured_smem[dev & 63] = (int)smem;
    }
    k_kgen<LG><<<H, T, smem, st>>>(Lambda, P, Q, B, C, log_dt, D, Nh, K, (float2 *)ws, flags);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_kgen(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B, const float2 *C,
                        const float *log_dt, const float *D, int H, int Nh, int L, float *K, void *ws,
                        unsigned *flags, cudaStream_t st) {
    switch (L) {
        case 16: return run_kgen<4>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 32: return run_kgen<5>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 64: return run_kgen<6>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 128: return run_kgen<7>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 256: return run_kgen<8>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 512: return run_kgen<9>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 1024: return run_kgen<10>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 2048: return run_kgen<11>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 4096: return run_kgen<12>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        case 8192: return run_kgen<13>(Lambda, P, Q, B, C, log_dt, D, H, Nh, K, ws, flags, st);
        default: {
            cudaError_t e = launch_cauchy(Lambda, P, Q, B, C, log_dt, H, Nh, L, K, flags, st);
            if (e == cudaSuccess) e = launch_kspec_from_half(K, D, H, L, ws, st);
            return e;
        }
    }
}

}  // namespace s4
