// cauchy.cuh -- the DPLR generating function at the roots of unity
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
// bin; sigma is taken back out of the sums at the end. The Nyquist bin
// z = -1 uses the limit K_hat(-1) = dt Re sum_n C_n B_n (the Woodbury term
// vanishes there).
#pragma once
#include "common.cuh"
#include "s4dplr.h"

namespace s4 {

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Per-mode constants of channel h into sp[3 n .. 3 n + 2] (nthreads threads):
// {m, rho, alpha00, beta00}, {alpha01, beta01, alpha10, beta10}, {alpha11, beta11, -, -}.
__device__ __forceinline__ void cauchy_stage_modes(const float2 *__restrict__ Lambda, const float2 *__restrict__ P,
                                                   const float2 *__restrict__ Q, const float2 *__restrict__ B,
                                                   const float2 *__restrict__ Cc, int h, int Nh, float4 *sp,
                                                   unsigned *flags, int tid, int nthreads) {
    const size_t pofs = (size_t)h * Nh;
    for (int n = tid; n < Nh; n += nthreads) {
        const float2 lam = Lambda[pofs + n], p = P[pofs + n], q = Q[pofs + n];
        const float2 b = B[pofs + n], c = Cc[pofs + n];
        const float2 v00 = cmul(c, b), v01 = cmul(c, p), v10 = cmulc(b, q), v11 = cmulc(p, q);
        auto be = [&](float2 v) { return 2.0f * fmaf(v.x, lam.x, v.y * lam.y); };  // 2 Re(v conj(lam))
        sp[3 * n + 0] = make_float4(fmaf(lam.x, lam.x, lam.y * lam.y), 2.0f * lam.x, 2.0f * v00.x, be(v00));
        sp[3 * n + 1] = make_float4(2.0f * v01.x, be(v01), 2.0f * v10.x, be(v10));
        sp[3 * n + 2] = make_float4(2.0f * v11.x, be(v11), 0.0f, 0.0f);
        if (flags != nullptr && !(lam.x < 0.0f)) atomicOr(flags, S4_FLAG_UNSTABLE);
    }
}

// K_hat at frequencies j[f] (0 <= j < L/2), times 1/L. inv_dt = 1/dt.
template <int F>
__device__ __forceinline__ void cauchy_eval(const float4 *sp, int Nh, const int (&j)[F], int L, float inv_dt,
                                            float2 (&kh)[F]) {
    float t[F], gam[F], sig[F], g2s[F], gs[F];
    float2 sb[F][4], sa[F][4];
#pragma unroll
    for (int f = 0; f < F; ++f) {
        float sn, cs;
        sincospif((float)j[f] / (float)L, &sn, &cs);   // j/L is exact, cs > 0 for j < L/2
        t[f] = __fdividef(sn, cs);
        gam[f] = 2.0f * t[f] * inv_dt;
        const float g2 = gam[f] * gam[f];
        // sigma = 2^-e with 2^(e-1) <= g2 < 2^e when g2 >= 1, else 1 (exact)
        const int e = ((__float_as_int(g2) >> 23) & 0xff) - 126;
        sig[f] = e > 0 ? __int_as_float((127 - e) << 23) : 1.0f;
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
    const float invL = 1.0f / (float)L;
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
        const float idn = rcp_approx(fmaf(den.x, den.x, den.y * den.y));
        const float2 w = cscale(cmulc(num, den), idn);
        const float2 r = csub(k[0], w);
        // times 2/(1+z) = 1 + i t, and 1/L for the inverse transform
        kh[f] = make_float2((r.x - t[f] * r.y) * invL, (r.y + t[f] * r.x) * invL);
    }
}

// K_hat at the Nyquist bin, times 1/L: dt Re sum_n C_n B_n / L (alpha00 / 2 summed)
__device__ __forceinline__ float cauchy_nyquist(const float4 *sp, int Nh, float dt, int L) {
    float acc = 0.0f;
    for (int n = 0; n < Nh; ++n) acc += sp[3 * n].z;
    return 0.5f * acc * dt / (float)L;
}

}  // namespace s4
