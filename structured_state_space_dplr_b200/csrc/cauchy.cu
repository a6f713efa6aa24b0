// cauchy.cu -- k_cauchy: the DPLR spectrum (four Cauchy sums, Woodbury,
// 2/(1+z); see cauchy.cuh), written packed into K itself:
//   K[0] = K_hat_0 (real), K[1] = K_hat_{L/2} (real), K[2j], K[2j+1] = K_hat_j,
// all times 1/L; k_irfft then turns it into the kernel in place.
#include "cauchy.cuh"
#include "launch.h"

namespace s4 {

// 128 threads x 4 frequencies per CTA (126 registers, four independent
// frequencies in flight per thread), the fastest of the shapes measured
// (CUDA events, H = 256: 21.0 us at L = 4096 and 66.7 us at L = 16384,
// against 21.3 / 70.6 us for 256 x 2, 21.6 / 70.7 for 128 x 2 and
// 21.3 / 68.5 for 64 x 4)
constexpr int kCauchyThreads = 128;
constexpr int kCauchyFreqs = 4;   // frequencies per thread

template <int T, int F>
__global__ void __launch_bounds__(T)
k_cauchy(const float2 *__restrict__ Lambda, const float2 *__restrict__ P, const float2 *__restrict__ Q,
         const float2 *__restrict__ B, const float2 *__restrict__ Cc, const float *__restrict__ log_dt,
         int Nh, int L, float *__restrict__ K, unsigned *__restrict__ flags) {
    extern __shared__ float4 sp[];
    const int h = blockIdx.y;
    cauchy_stage_modes<true>(Lambda, P, Q, B, Cc, h, Nh, sp, flags, threadIdx.x, T);
    __syncthreads();
    const float ldt = __ldg(log_dt + h);
    const int half = L >> 1;
    int j[F], jj[F];
#pragma unroll
    for (int f = 0; f < F; ++f) {
        j[f] = blockIdx.x * (T * F) + f * T + threadIdx.x;
        jj[f] = j[f] < half ? j[f] : 0;
    }
    float2 kh[F];
    cauchy_eval<F, true>(sp, Nh, jj, L, expf(-ldt), kh);
    bool bad = false;
    float *Kh = K + (size_t)h * L;
#pragma unroll
    for (int f = 0; f < F; ++f) {
        if (j[f] < half) {
            if (j[f] == 0) Kh[0] = kh[f].x;
            else *reinterpret_cast<float2 *>(Kh + 2 * j[f]) = kh[f];
            bad |= !(isfinite(kh[f].x) && isfinite(kh[f].y));
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        const float nyq = cauchy_nyquist<true>(sp, Nh, expf(ldt), L);
        Kh[1] = nyq;
        bad |= !isfinite(nyq);
    }
    if (flags != nullptr && __any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
        atomicOr(flags, S4_FLAG_NONFINITE);
}

cudaError_t launch_cauchy(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B,
                          const float2 *C, const float *log_dt, int H, int Nh, int L, float *K,
                          unsigned *flags, cudaStream_t st) {
    constexpr int T = kCauchyThreads, F = kCauchyFreqs;
    const int half = L / 2;
    dim3 grid((half + T * F - 1) / (T * F), H);
    const size_t smem = sizeof(float4) * cauchy_mode_words<true>() * (size_t)Nh;
    k_cauchy<T, F><<<grid, T, smem, st>>>(Lambda, P, Q, B, C, log_dt, Nh, L, K, flags);
    return cudaGetLastError();
}

}  // namespace s4
