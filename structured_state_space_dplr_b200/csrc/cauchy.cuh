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

// Two forms of the mode loop, each chosen where it measured faster: scalar
// FP32 instructions, or sm_100's paired FP32 instructions (__ffma2_rn: two
// independent fused multiply-adds per issued instruction, each rounded as
// fmaf). The paired form halves the instructions issued but lengthens the
// dependency chains, which pays in a kernel with many resident warps
// (k_cauchy) and costs in one with few (k_kgen).
//
// Words (float4) of staged constants per mode for each form.
template <bool PAIRED>
__host__ __device__ constexpr int cauchy_mode_words() { return PAIRED ? 5 : 3; }

// Per-mode constants of channel h into sp[W n .. W n + W - 1] (nthreads
// threads), W = cauchy_mode_words<PAIRED>(), a = alpha_v, b = beta_v:
//   scalar: {m, rho, a00, b00}, {a01, b01, a10, b10}, {a11, b11, -, -};
//   paired: {m, rho, b00, b00}, {a00, a00, b01, b01}, {a01, a01, b10, b10},
//           {a10, a10, b11, b11}, {a11, a11, -, -} -- each coefficient twice,
//           side by side, so it reaches the paired instructions as an
//           aligned register pair.
template <bool PAIRED>
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
        const float a00 = 2.0f * v00.x, a01 = 2.0f * v01.x, a10 = 2.0f * v10.x, a11 = 2.0f * v11.x;
        const float b00 = be(v00), b01 = be(v01), b10 = be(v10), b11 = be(v11);
        const float m = fmaf(lam.x, lam.x, lam.y * lam.y), rho = 2.0f * lam.x;
        float4 *w = sp + cauchy_mode_words<PAIRED>() * n;
        if constexpr (PAIRED) {
            w[0] = make_float4(m, rho, b00, b00);
            w[1] = make_float4(a00, a00, b01, b01);
            w[2] = make_float4(a01, a01, b10, b10);
            w[3] = make_float4(a10, a10, b11, b11);
            w[4] = make_float4(a11, a11, 0.0f, 0.0f);
        } else {
            w[0] = make_float4(m, rho, a00, b00);
            w[1] = make_float4(a01, b01, a10, b10);
            w[2] = make_float4(a11, b11, 0.0f, 0.0f);
        }
        if (flags != nullptr && !(lam.x < 0.0f)) atomicOr(flags, S4_FLAG_UNSTABLE);
    }
}

// K_hat at frequencies j[f] (0 <= j < L/2), times 1/L. inv_dt = 1/dt.
// Per mode and frequency: the scaled denominator q = sigma (m - gamma^2,
// rho gamma), r = 1/q, and the four sums {S_beta r, S_alpha r} accumulated
// over the complex r.
template <int F, bool PAIRED>
__device__ __forceinline__ void cauchy_eval(const float4 *sp, int Nh, const int (&j)[F], int L, float inv_dt,
                                            float2 (&kh)[F]) {
    float t[F], gam[F], sig[F];
    float2 sg[F], ng[F];        // {sigma, gamma sigma}, {-gamma^2 sigma, 0}
    float2 sb[F][4], sa[F][4];  // {sum beta_v re r, sum beta_v im r}, same for alpha_v
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
        sg[f] = make_float2(sig[f], gam[f] * sig[f]);
        ng[f] = make_float2(-(g2 * sig[f]), 0.0f);
#pragma unroll
        for (int v = 0; v < 4; ++v) { sb[f][v] = make_float2(0.f, 0.f); sa[f][v] = make_float2(0.f, 0.f); }
    }
#pragma unroll 2
    for (int n = 0; n < Nh; ++n) {
        const float4 *w = sp + cauchy_mode_words<PAIRED>() * n;
        if constexpr (PAIRED) {
            const float4 w0 = w[0], w1 = w[1], w2 = w[2], w3 = w[3], w4 = w[4];
            const float2 mr = make_float2(w0.x, w0.y);
            const float2 bt[4] = {make_float2(w0.z, w0.w), make_float2(w1.z, w1.w), make_float2(w2.z, w2.w),
                                  make_float2(w3.z, w3.w)};
            const float2 al[4] = {make_float2(w1.x, w1.y), make_float2(w2.x, w2.y), make_float2(w3.x, w3.y),
                                  make_float2(w4.x, w4.y)};
#pragma unroll
            for (int f = 0; f < F; ++f) {
                const float2 q = __ffma2_rn(mr, sg[f], ng[f]);
                const float inv = rcp_approx(fmaf(q.x, q.x, q.y * q.y));
                const float2 r = make_float2(q.x * inv, q.y * inv);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    sb[f][v] = __ffma2_rn(bt[v], r, sb[f][v]);
                    sa[f][v] = __ffma2_rn(al[v], r, sa[f][v]);
                }
            }
        } else {
            const float4 a = w[0], b = w[1], c = w[2];
            const float al[4] = {a.z, b.x, b.z, c.x};
            const float bt[4] = {a.w, b.y, b.w, c.y};
#pragma unroll
            for (int f = 0; f < F; ++f) {
                const float qx = fmaf(a.x, sg[f].x, ng[f].x), qy = a.y * sg[f].y;
                const float inv = rcp_approx(fmaf(qx, qx, qy * qy));
                const float rr = qx * inv, ri = qy * inv;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    sb[f][v].x = fmaf(bt[v], rr, sb[f][v].x);
                    sb[f][v].y = fmaf(bt[v], ri, sb[f][v].y);
                    sa[f][v].x = fmaf(al[v], rr, sa[f][v].x);
                    sa[f][v].y = fmaf(al[v], ri, sa[f][v].y);
                }
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
template <bool PAIRED>
__device__ __forceinline__ float cauchy_nyquist(const float4 *sp, int Nh, float dt, int L) {
    float acc = 0.0f;
    for (int n = 0; n < Nh; ++n) acc += PAIRED ? sp[5 * n + 1].x : sp[3 * n].z;
    return 0.5f * acc * dt / (float)L;
}

}  // namespace s4
