// cauchy.cu -- the DPLR generating function at the roots of unity
// ("The S4 kernel, from scratch", §4): four Cauchy sums over the modes, the
// rank-1 Woodbury correction and the bilinear factor 2/(1+z).
//
// At z_j = exp(-2 pi i j/L) the bilinear map gives g(z_j) = (2/dt)(1-z)/(1+z)
// = i gamma_j with gamma_j = (2/dt) tan(pi j/L), and 2/(1+z_j) = 1 + i t_j,
// t_j = tan(pi j/L). A stored mode n and its implicit conjugate contribute
// together (v = C B, C P, conj(Q) B or conj(Q) P):
//   v/(g - Lambda) + conj(v)/(g - conj(Lambda))
//       = (-beta_v + i alpha_v gamma) / ((m - gamma^2) - i rho gamma),
//   alpha_v = 2 Re v,  beta_v = 2 Re(v conj(Lambda)),  m = |Lambda|^2,
//   rho = 2 Re Lambda.
// So with r_n = 1/((m - gamma^2) - i rho gamma) each Cauchy sum is
//   k_v = -sum_n beta_v r_n + i gamma sum_n alpha_v r_n,
// which costs one reciprocal and 16 FMAs per mode pair for all four sums.
// The denominator is scaled by a power of two sigma ~ 1/gamma^2 per frequency
// (exact, it only shifts exponents) so it stays in range up to the Nyquist
// bin; sigma is taken back out of the sums at the end.
//
// The spectrum K_hat_j (j = 0 .. L/2, times 1/L for the inverse transform) is
// written packed into K itself: K[0] = K_hat_0 (real), K[1] = K_hat_{L/2}
// (real), K[2j], K[2j+1] = Re, Im K_hat_j; the inverse real FFT then turns
// it into the kernel in place. The Nyquist bin z = -1 uses the limit
// K_hat(-1) = dt Re sum_n C_n B_n (the Woodbury term vanishes there).
#include "common.cuh"
#include "launch.h"
#include "s4dplr.h"

namespace s4 {

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

constexpr int kCauchyThreads = 256;
constexpr int kCauchyFreqs = 2;   // frequencies per thread

template <int T, int F>
__global__ void __launch_bounds__(T)
k_cauchy(const float2 *__restrict__ Lambda, const float2 *__restrict__ P, const float2 *__restrict__ Q,
         const float2 *__restrict__ B, const float2 *__restrict__ Cc, const float *__restrict__ log_dt,
         int Nh, int L, float *__restrict__ K, unsigned *__restrict__ flags) {
    extern __shared__ float4 sp[];   // [Nh][3]: {m, rho, a00, b00}, {a01, b01, a10, b10}, {a11, b11, -, -}
    const int h = blockIdx.y;
    const size_t pofs = (size_t)h * Nh;
    for (int n = threadIdx.x; n < Nh; n += T) {
        const float2 lam = Lambda[pofs + n], p = P[pofs + n], q = Q[pofs + n];
        const float2 b = B[pofs + n], c = Cc[pofs + n];
        const float2 v00 = cmul(c, b), v01 = cmul(c, p), v10 = cmulc(b, q), v11 = cmulc(p, q);
        auto be = [&](float2 v) { return 2.0f * fmaf(v.x, lam.x, v.y * lam.y); };  // 2 Re(v conj(lam))
        sp[3 * n + 0] = make_float4(fmaf(lam.x, lam.x, lam.y * lam.y), 2.0f * lam.x, 2.0f * v00.x, be(v00));
        sp[3 * n + 1] = make_float4(2.0f * v01.x, be(v01), 2.0f * v10.x, be(v10));
        sp[3 * n + 2] = make_float4(2.0f * v11.x, be(v11), 0.0f, 0.0f);
        if (flags != nullptr && !(lam.x < 0.0f)) atomicOr(flags, S4_FLAG_UNSTABLE);
    }
    __syncthreads();

    const float ldt = __ldg(log_dt + h);
    const float inv_dt = expf(-ldt);
    const int half = L >> 1;
    const float invL = 1.0f / (float)L;

    int j[F];
    float t[F], gam[F], sig[F], g2s[F], gs[F];
    float2 sb[F][4], sa[F][4];
#pragma unroll
    for (int f = 0; f < F; ++f) {
        j[f] = blockIdx.x * (T * F) + f * T + threadIdx.x;
        const int jj = j[f] < half ? j[f] : 0;
        float sn, cs;
        sincospif((float)jj / (float)L, &sn, &cs);
        t[f] = sn / cs;
        gam[f] = 2.0f * t[f] * inv_dt;
        const float g2 = gam[f] * gam[f];
        int e;
        frexpf(g2, &e);
        sig[f] = e > 0 ? ldexpf(1.0f, -e) : 1.0f;
        g2s[f] = g2 * sig[f];
        gs[f] = gam[f] * sig[f];
#pragma unroll
        for (int v = 0; v < 4; ++v) { sb[f][v] = make_float2(0.f, 0.f); sa[f][v] = make_float2(0.f, 0.f); }
    }

#pragma unroll 2
    for (int n = 0; n < Nh; ++n) {
        const float4 a = sp[3 * n + 0], b = sp[3 * n + 1], c = sp[3 * n + 2];
        const float al[4] = {a.z, b.x, b.z, c.x};
        const float bt[4] = {a.w, b.y, b.w, c.y};
#pragma unroll
        for (int f = 0; f < F; ++f) {
            const float A = fmaf(a.x, sig[f], -g2s[f]);
            const float Bq = a.y * gs[f];
            const float Dn = fmaf(A, A, Bq * Bq);
            const float inv = rcp_approx(Dn);
            const float rr = A * inv, ri = Bq * inv;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                sb[f][v].x = fmaf(bt[v], rr, sb[f][v].x);
                sb[f][v].y = fmaf(bt[v], ri, sb[f][v].y);
                sa[f][v].x = fmaf(al[v], rr, sa[f][v].x);
                sa[f][v].y = fmaf(al[v], ri, sa[f][v].y);
            }
        }
    }

    bool bad = false;
#pragma unroll
    for (int f = 0; f < F; ++f) {
        float2 k[4];
#pragma unroll
        for (int v = 0; v < 4; ++v)   // k_v = sigma (-S_beta + i gamma S_alpha)
            k[v] = make_float2(sig[f] * (-sb[f][v].x - gam[f] * sa[f][v].y),
                               sig[f] * (-sb[f][v].y + gam[f] * sa[f][v].x));
        // Woodbury: k00 - k01 k10 / (1 + k11)
        const float2 den = make_float2(1.0f + k[3].x, k[3].y);
        const float2 num = cmul(k[1], k[2]);
        const float idn = 1.0f / fmaf(den.x, den.x, den.y * den.y);
        const float2 w = cscale(cmulc(num, den), idn);
        const float2 r = csub(k[0], w);
        // times 2/(1+z) = 1 + i t, and 1/L for the inverse transform
        const float2 kh = make_float2((r.x - t[f] * r.y) * invL, (r.y + t[f] * r.x) * invL);
        if (j[f] < half) {
            float *Kh = K + (size_t)h * L;
            if (j[f] == 0) {
                Kh[0] = kh.x;
            } else {
                *reinterpret_cast<float2 *>(Kh + 2 * j[f]) = kh;
            }
            bad |= !(isfinite(kh.x) && isfinite(kh.y));
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        float acc = 0.0f;   // sum_n alpha_00 / 2 = Re sum_n C_n B_n
        for (int n = 0; n < Nh; ++n) acc += sp[3 * n].z;
        const float nyq = 0.5f * acc * expf(ldt) * invL;
        K[(size_t)h * L + 1] = nyq;
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
    const size_t smem = sizeof(float4) * 3 * (size_t)Nh;
    k_cauchy<T, F><<<grid, T, smem, st>>>(Lambda, P, Q, B, C, log_dt, Nh, L, K, flags);
    return cudaGetLastError();
}

}  // namespace s4
