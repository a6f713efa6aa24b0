// kgen.cu -- the DPLR kernel K and the spectrum of the zero-padded K + D
// delta_0 in one launch ("The S4 kernel, from scratch", §4 and §5), for
// L <= 4096. One CTA per channel:
//   A. the Cauchy/Woodbury generating function at j = 0 .. L/2 (cauchy.cuh),
//      written with its conjugate mirror straight into the digit-reversed
//      positions the inverse transform reads;
//   B. length-L inverse transform (decimation in time) -> K, stored;
//   C. the same registers start the length-2L forward transform of the
//      zero-padded K (both halves of the transform, as in k_fftconv_pair);
//      its spectrum, plus D and times 1/2L, goes to the convolution workspace
//      in the layout k_fftconv_pair reads.
// Longer kernels take the three-kernel path (k_cauchy, k_irfft, k_kspec).
#include "cauchy.cuh"
#include "fft.cuh"
#include "launch.h"

namespace s4 {

template <int LG>
__host__ __device__ constexpr int kgen_threads() { return (1 << LG) / 16 < 32 ? 32 : (1 << LG) / 16; }

// shared memory in float4: X, Y (padded m float2 each) | tws | ta, tb | modes
template <int LG>
__host__ __device__ constexpr int kgen_smem_f2() {
    return 2 * padded(1 << LG) + plan_tw_size(LG) + 2 * ((1 << LG) >> plan_lr(LG, 0));
}

template <int LG>
__global__ void __launch_bounds__(kgen_threads<LG>(), 2)
k_kgen(const float2 *__restrict__ Lambda, const float2 *__restrict__ P, const float2 *__restrict__ Q,
       const float2 *__restrict__ B, const float2 *__restrict__ Cc, const float *__restrict__ log_dt,
       const float *__restrict__ D, int Nh, float *__restrict__ K, float2 *__restrict__ spec,
       unsigned *__restrict__ flags) {
    constexpr int m = 1 << LG, L = m, T = kgen_threads<LG>(), N = 2 * m;
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0, NP = plan_P(LG);
    constexpr int F = 4;   // frequencies per thread per round
    extern __shared__ float4 smem4[];
    float2 *X = reinterpret_cast<float2 *>(smem4), *Y = X + padded(m);
    float2 *tws = Y + padded(m);
    float2 *ta = tws + plan_tw_size(LG), *tb = ta + S0;
    float4 *sp = reinterpret_cast<float4 *>(X + ((kgen_smem_f2<LG>() + 1) / 2) * 2);
    const int h = blockIdx.x;

    for (int i = threadIdx.x; i < S0; i += T) {
        ta[i] = unit_root(i, N);
        tb[i] = unit_root(i, m);
    }
    build_middle_tables<LG>(tws, threadIdx.x, T);
    cauchy_stage_modes(Lambda, P, Q, B, Cc, h, Nh, sp, flags, threadIdx.x, T);
    __syncthreads();

    // ---- A: generating function -> X at digit-reversed positions (with mirror)
    const float ldt = __ldg(log_dt + h);
    const float inv_dt = expf(-ldt);
    bool bad = false;
    for (int f0 = 0; f0 < L / 2; f0 += T * F) {
        int j[F], jj[F];
#pragma unroll
        for (int f = 0; f < F; ++f) {
            j[f] = f0 + f * T + threadIdx.x;
            jj[f] = j[f] < L / 2 ? j[f] : 0;
        }
        float2 kh[F];
        cauchy_eval<F>(sp, Nh, jj, L, inv_dt, kh);
#pragma unroll
        for (int f = 0; f < F; ++f) {
            if (j[f] < L / 2) {
                bad |= !(isfinite(kh[f].x) && isfinite(kh[f].y));
                if (j[f] == 0) {
                    X[pidx(0)] = make_float2(kh[f].x, 0.0f);
                } else {
                    X[pidx(digrev_inv<LG>(j[f]))] = kh[f];
                    X[pidx(digrev_inv<LG>(L - j[f]))] = cconj(kh[f]);
                }
            }
        }
    }
    if (threadIdx.x == 0) {
        const float nyq = cauchy_nyquist(sp, Nh, expf(ldt), L);
        bad |= !isfinite(nyq);
        X[pidx(digrev_inv<LG>(L / 2))] = make_float2(nyq, 0.0f);
    }
    if (flags != nullptr && __any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
        atomicOr(flags, S4_FLAG_NONFINITE);
    __syncthreads();

    // ---- B: inverse transform, passes P-1 .. 1
    dit_pass<LG, NP - 1, +1, T>(X, tws);
    __syncthreads();
    inverse_middle<LG, T>(X, tws);

    // ---- B/C: last inverse pass -> K (stored), first forward pass of both halves
    float *Kh = K + (size_t)h * L;
    for (int j = threadIdx.x; j < S0; j += T) {
        const int o = pidx(j);
        const float2 a = ta[j], b = tb[j];
        float2 x[R0], z[R0];
        {
            float2 w = b;
            x[0] = X[o];
            static_for<1, R0>([&](auto q) {
                x[q] = cmulc(X[o + poff<decltype(q)::value * S0>()], w);
                w = cmul(w, b);
            });
        }
        dft<R0, +1>(x);
        static_for<0, R0>([&](auto p) {
            const float k = x[p].x;   // K is real: the imaginary part is rounding
            Kh[j + p * S0] = k;
            x[p] = make_float2(k, 0.0f);
            z[p] = rot<decltype(p)::value, 2 * R0, -1>(x[p]);
        });
        dft<R0, -1>(x);
        dft<R0, -1>(z);
        float2 w = b, v = a;
        X[o] = x[0];
        Y[o] = cmul(z[0], a);
        static_for<1, R0>([&](auto q) {
            v = cmul(v, b);
            X[o + poff<decltype(q)::value * S0>()] = cmul(x[q], w);
            Y[o + poff<decltype(q)::value * S0>()] = cmul(z[q], v);
            w = cmul(w, b);
        });
    }
    __syncthreads();

    // ---- C: forward passes 1 .. P-2, last pass -> (spectrum + D) / 2L
    forward_middle_x2<LG, T>(X, Y, tws);
    const float Dh = D != nullptr ? __ldg(D + h) : 0.0f;
    const float scale = 1.0f / (float)N;
    constexpr int lr = plan_lr(LG, NP - 1), R = 1 << lr;
    float4 *o0 = reinterpret_cast<float4 *>(spec + (size_t)h * N);
    float4 *o1 = o0 + m / 2;
    for (int g = threadIdx.x; g < m / R; g += T) {
        const int base = g * R, o = pidx(base);
        float2 x[R], z[R];
        load_contig<R>(X + o, x);
        load_contig<R>(Y + o, z);
        dft<R, -1>(x);
        dft<R, -1>(z);
        static_for<0, R / 2>([&](auto i) {
            o0[spec4_index<LG>(base, i)] = make_float4((x[2 * i].x + Dh) * scale, x[2 * i].y * scale,
                                           (x[2 * i + 1].x + Dh) * scale, x[2 * i + 1].y * scale);
            o1[spec4_index<LG>(base, i)] = make_float4((z[2 * i].x + Dh) * scale, z[2 * i].y * scale,
                                           (z[2 * i + 1].x + Dh) * scale, z[2 * i + 1].y * scale);
        });
    }
}

namespace {
template <int LG>
cudaError_t run_kgen(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B, const float2 *C,
                     const float *log_dt, const float *D, int H, int Nh, float *K, void *ws, unsigned *flags,
                     cudaStream_t st) {
    constexpr int T = kgen_threads<LG>();
    const size_t smem = sizeof(float2) * (size_t)((kgen_smem_f2<LG>() + 1) / 2 * 2) + sizeof(float4) * 3 * (size_t)Nh;
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
        default: {
            cudaError_t e = launch_cauchy(Lambda, P, Q, B, C, log_dt, H, Nh, L, K, flags, st);
            if (e == cudaSuccess) e = launch_irfft_packed(K, H, L, st);
            if (e == cudaSuccess) e = launch_kspec(K, D, H, L, ws, st);
            return e;
        }
    }
}

}  // namespace s4
