// backward.cu -- gradients of the convolution view ("The S4 kernel, from
// scratch", §5 fft_conv; §6 makes the layer trainable) for L <= 8192:
//
//   du[b,h,s] = sum_{t>=s} K[h,t-s] dy[b,h,t] + D[h] dy[b,h,s]
//             -- the forward convolution kernel with the conjugate spectrum
//                (k_fftconv_pair<LG, true>, spectral.cu);
//   dK[h,k]   = sum_b sum_{t>=k} dy[b,h,t] u[b,h,t-k],   dD[h] = dK[h,0]
//             -- k_corr_pair below.
//
// dK: two rows are packed as for the forward, Zu = FFT_2L(u_b + i u_b+1) and
// Zd = FFT_2L(dy_b + i dy_b+1). With U, D the spectra of the single rows,
//   conj(Zu) Zd = conj(U_b) D_b + conj(U_b+1) D_b+1
//               + i (conj(U_b) D_b+1 - conj(U_b+1) D_b),
// and the inverse transform of each bracket is a real correlation: the two
// wanted correlations land in the real part, the cross terms in the imaginary
// part. So conj(Zu) Zd is summed over the row pairs of a channel (in the
// digit-reversed order the forward passes leave, no reordering) and inverse
// transformed once; the real part of the first L outputs, times 1/2L, is dK.
#include "launch.h"
#include "pairs.cuh"

namespace s4 {

// One CTA per channel at a time (persistent over channels), looping over the
// channel's row pairs. The forward transform of the u pair leaves Zu in the
// channel's scratch slice, that of the dy pair multiplies its last-pass
// groups by conj(Zu) and accumulates into the channel's acc slice; each
// thread owns the same last-pass groups throughout, so the scratch and the
// accumulator are read back only by the thread that wrote them.
template <int LG>
__global__ void __launch_bounds__(pair_threads<LG>(), pair_min_blocks<LG>())
k_corr_pair(const float *__restrict__ u, const float *__restrict__ dy, int Bt, int H, float *__restrict__ dK,
            float *__restrict__ dD, float2 *__restrict__ acc, float2 *__restrict__ zs) {
    constexpr int m = 1 << LG, L = m, T = pair_threads<LG>();
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    constexpr int RL = 1 << plan_lr(LG, plan_P(LG) - 1), G = m / RL;
    extern __shared__ float2 sm[];
    const PairSmem s = pair_carve<LG>(sm);
    pair_tables<LG>(s);
    __syncthreads();
    const int nbp = (Bt + 1) / 2;
    for (int h = blockIdx.x; h < H; h += gridDim.x) {
        float4 *A0 = reinterpret_cast<float4 *>(acc + (size_t)h * 2 * m), *A1 = A0 + m / 2;
        float4 *Z0 = reinterpret_cast<float4 *>(zs + (size_t)h * 2 * m), *Z1 = Z0 + m / 2;
        for (int bp = 0; bp < nbp; ++bp) {
            const int b0 = 2 * bp;
            const bool has1 = b0 + 1 < Bt;
#pragma unroll 1
            for (int pass = 0; pass < 2; ++pass) {   // 0: u pair -> Zu; 1: dy pair -> acc
                const float *r0 = (pass == 0 ? u : dy) + ((size_t)b0 * H + h) * L;
                const float *r1 = r0 + (size_t)H * L;
                for (int j = threadIdx.x; j < S0; j += T) {
                    float2 v[R0];
                    static_for<0, R0>([&](auto p) {
                        const int k = j + p * S0;
                        v[p] = make_float2(__ldg(r0 + k), has1 ? __ldg(r1 + k) : 0.0f);
                    });
                    first_pass_halves<LG>(s, v, j);
                }
                __syncthreads();
                forward_middle_x2<LG, T>(s.b0, s.b1, s.tws);
                for (int g = threadIdx.x; g < G; g += T) {
                    const int base = g * RL, o = pidx(base);
                    float2 x[RL], z[RL];
                    load_contig<RL>(s.b0 + o, x);
                    load_contig<RL>(s.b1 + o, z);
                    dft<RL, -1>(x);
                    dft<RL, -1>(z);
                    static_for<0, RL / 2>([&](auto i) {
                        const int w = spec4_index<LG>(base, i);
                        const float2 x0 = x[2 * i], x1 = x[2 * i + 1], z0 = z[2 * i], z1 = z[2 * i + 1];
                        if (pass == 0) {
                            Z0[w] = make_float4(x0.x, x0.y, x1.x, x1.y);
                            Z1[w] = make_float4(z0.x, z0.y, z1.x, z1.y);
                        } else {
                            const float4 u0 = Z0[w], u1 = Z1[w];
                            const float2 p0 = cmulc(x0, make_float2(u0.x, u0.y));   // Zd conj(Zu)
                            const float2 p1 = cmulc(x1, make_float2(u0.z, u0.w));
                            const float2 q0 = cmulc(z0, make_float2(u1.x, u1.y));
                            const float2 q1 = cmulc(z1, make_float2(u1.z, u1.w));
                            float4 a0 = make_float4(p0.x, p0.y, p1.x, p1.y);
                            float4 a1 = make_float4(q0.x, q0.y, q1.x, q1.y);
                            if (bp > 0) {
                                const float4 c0 = A0[w], c1 = A1[w];
                                a0 = make_float4(a0.x + c0.x, a0.y + c0.y, a0.z + c0.z, a0.w + c0.w);
                                a1 = make_float4(a1.x + c1.x, a1.y + c1.y, a1.z + c1.z, a1.w + c1.w);
                            }
                            A0[w] = a0;
                            A1[w] = a1;
                        }
                    });
                }
                __syncthreads();   // the buffers are transformed again next
            }
        }
        // ---- inverse transform of the accumulated product, both halves
        for (int g = threadIdx.x; g < G; g += T) {
            const int base = g * RL, o = pidx(base);
            float2 x[RL], z[RL];
            static_for<0, RL / 2>([&](auto i) {
                const int w = spec4_index<LG>(base, i);
                const float4 c0 = A0[w], c1 = A1[w];
                x[2 * i] = make_float2(c0.x, c0.y);
                x[2 * i + 1] = make_float2(c0.z, c0.w);
                z[2 * i] = make_float2(c1.x, c1.y);
                z[2 * i + 1] = make_float2(c1.z, c1.w);
            });
            dft<RL, +1>(x);
            dft<RL, +1>(z);
            store_contig<RL>(s.b0 + o, x);
            store_contig<RL>(s.b1 + o, z);
        }
        __syncthreads();
        inverse_middle_x2<LG, T>(s.b0, s.b1, s.tws);
        const float scale = 1.0f / (float)(2 * m);
        float *dKh = dK + (size_t)h * L;
        last_pass_halves_sum<LG>(s, [&](auto, int t, float2 r, float2) {
            dKh[t] = r.x * scale;
            if (t == 0 && dD != nullptr) dD[h] = r.x * scale;
        });
        __syncthreads();   // the buffers are reused by the next channel
    }
}

// ------------------------------------------------------ kernel parameters --
// Gradient of a loss through K = iDFT(K_hat) with respect to the DPLR
// parameters ("The S4 kernel, from scratch", §4 generating function, §6
// trainable parameters), given dK = dLoss/dK [H, L].
//
// With G_hat = DFT(dK), the loss moves with K_hat_j (j < L/2, each with its
// Hermitian partner) through g_j = dLoss/dRe K_hat_j + i dLoss/dIm K_hat_j
// = (2/L) G_hat_j ((1/L) G_hat_0 at j = 0). K_hat_j = c_j R_j with
// c_j = 1 + i t_j, R = k00 - k01 k10 / (1 + k11) and
// k_v = sum_i v_i r_i over the full conjugate-closed system,
// r_i = 1/(s_j - lambda_i), s_j = i gamma_j. Writing e_v = dK_hat/dk_v
// (e00 = c, e01 = -c k10/(1+k11), e10 = -c k01/(1+k11),
// e11 = c k01 k10/(1+k11)^2) and a_v = conj(g_j) e_v, every complex
// parameter's gradient (d/dRe + i d/dIm) of a stored mode n collects, per v,
//   S_v  = sum_j a_v r_n' + conj(a_v r_n)         (r_n' = 1/(s - conj lambda_n))
//   S2_v = sum_j a_v r_n'^2 + conj(a_v r_n^2),
// and then
//   dC = conj(B) S00 + conj(P) S01,   dB = conj(C) S00 + Q S10,
//   dP = conj(C) S01 + Q S11,         dQ = B conj(S10) + P conj(S11),
//   dLambda = sum_v conj(v_v) S2_v    (v00 = CB, v01 = CP, v10 = conj(Q) B,
//                                      v11 = conj(Q) P);
//   dlog_dt = sum_j Re(conj(g_j) s_j sum_v e_v sum_i v_i r_i^2)
// (s_j scales as 1/dt). The Nyquist bin, K_hat = dt Re sum_n C_n B_n, adds
// g dt conj(B) to dC, g dt conj(C) to dB and g K_hat to dlog_dt.
//
// One CTA per channel (persistent): G_hat by a length-L forward transform in
// shared memory; then frequencies in chunks of T: each thread forms the four
// k_v and sum_i v_i r_i^2 of one frequency (its a_v go to shared memory),
// then thread (n, q) accumulates S_v, S2_v of mode n over every nq-th
// frequency of the chunk; the nq partial sums of a mode are added at the end.
constexpr int kBwdThreads = 256;
constexpr int kModeFloats = 20;   // lambda(2) C(2) B(2) P(2) Q(2) v00..v11(8) -(2)

// GG: G_hat comes from global memory (computed by the four-step DFT below), no
// transform in shared memory
template <int LG, bool GG>
__host__ __device__ constexpr size_t kbwd_smem_bytes(int Nh) {
    return (GG ? 0
               : sizeof(float2) * ((size_t)padded(1 << LG) + plan_tw_size(LG) + ((1 << LG) >> plan_lr(LG, 0)))) +
           sizeof(float) * ((size_t)kModeFloats * Nh + 9 * kBwdThreads + 16 * kBwdThreads + 32);
}

// 1/d for complex d (hardware reciprocal of |d|^2; |d| >= |Re lambda| > 0)
__device__ __forceinline__ float2 crcp(float2 d) {
    float inv;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(fmaf(d.x, d.x, d.y * d.y)));
    return make_float2(d.x * inv, -d.y * inv);
}

template <int LG, bool GG>
__global__ void __launch_bounds__(kBwdThreads, 2)
k_kgen_backward(const float2 *__restrict__ Lambda, const float2 *__restrict__ P, const float2 *__restrict__ Q,
                const float2 *__restrict__ B, const float2 *__restrict__ Cc, const float *__restrict__ log_dt,
                const float *__restrict__ dK, const float2 *__restrict__ ghat, int H, int Nh, int FS,
                float *__restrict__ part, float2 *__restrict__ dLambda, float2 *__restrict__ dP,
                float2 *__restrict__ dQ, float2 *__restrict__ dB, float2 *__restrict__ dC,
                float *__restrict__ dlog_dt) {
    constexpr int m = 1 << LG, L = m, T = kBwdThreads;
    constexpr int R0 = 1 << plan_lr(LG, 0), S0 = m / R0;
    constexpr int RL = 1 << plan_lr(LG, plan_P(LG) - 1);
    extern __shared__ float2 smb[];
    float2 *buf = smb, *tws = buf + (GG ? 0 : padded(m)), *tb = tws + (GG ? 0 : plan_tw_size(LG));
    float *md = reinterpret_cast<float *>(tb + (GG ? 0 : S0));   // [Nh][kModeFloats]
    float *chA = md + kModeFloats * Nh;                      // [T][8]  a_v of the chunk
    float *chG = chA + 8 * T;                                // [T]     gamma of the chunk
    float *red = chG + T;                                    // [T][16] partial sums
    float *red32 = red + 16 * T;                             // [32]
    const int tid = threadIdx.x;
    if constexpr (!GG) {
        for (int j = tid; j < S0; j += T) tb[j] = unit_root(j, m);
        build_middle_tables<LG>(tws, tid, T);
    }
    const int nq = T / Nh;   // frequency slices per mode (Nh <= T)
    const int my_n = tid % Nh, my_q = tid / Nh;

    // GG: item = (channel, frequency slice f of FS); the slice's per-mode
    // sums go to part[item] and k_kgen_backward_assemble adds the slices
    const int nitems = GG ? H * FS : H;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
        const int h = GG ? item / FS : item;
        const int jb = GG ? (int)((long long)(L / 2) * (item % FS) / FS) : 0;
        const int je = GG ? (int)((long long)(L / 2) * (item % FS + 1) / FS) : L / 2;
        const size_t po = (size_t)h * Nh;
        const float dt = expf(__ldg(log_dt + h));
        for (int n = tid; n < Nh; n += T) {
            const float2 lam = Lambda[po + n], c = Cc[po + n], b = B[po + n], p = P[po + n], q = Q[po + n];
            const float2 v00 = cmul(c, b), v01 = cmul(c, p), v10 = cmulc(b, q), v11 = cmulc(p, q);
            float *w = md + kModeFloats * n;
            const float vals[kModeFloats] = {lam.x, lam.y, c.x, c.y, b.x, b.y, p.x, p.y, q.x, q.y,
                                             v00.x, v00.y, v01.x, v01.y, v10.x, v10.y, v11.x, v11.y, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < kModeFloats; ++i) w[i] = vals[i];
        }
        // ---- G_hat = DFT(dK): forward transform, digit-reversed result in buf
        const float *dKh = dK + (size_t)h * L;
        if constexpr (!GG) {
        for (int j = tid; j < S0; j += T) {
            float2 x[R0];
            static_for<0, R0>([&](auto p) { x[p] = make_float2(__ldg(dKh + j + p * S0), 0.0f); });
            dft<R0, -1>(x);
            const float2 b = tb[j];
            float2 w = b;
            float2 *o = buf + pidx(j);
            o[0] = x[0];
            static_for<1, R0>([&](auto q) {
                o[poff<decltype(q)::value * S0>()] = cmul(x[q], w);
                w = cmul(w, b);
            });
        }
        __syncthreads();
        forward_middle<LG, T>(buf, tws);
        for (int g = tid; g < m / RL; g += T) {
            float2 x[RL];
            float2 *o = buf + pidx(g * RL);
            load_contig<RL>(o, x);
            dft<RL, -1>(x);
            store_contig<RL>(o, x);
        }
        }   // !GG
        __syncthreads();
        const float2 *gh = ghat + (size_t)h * (L / 2 + 1);

        float ld_acc = 0.0f;
        float2 S[4], S2[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) S[v] = S2[v] = make_float2(0.f, 0.f);
        const float2 lam_n = make_float2(md[kModeFloats * my_n], md[kModeFloats * my_n + 1]);
        for (int j0 = jb; j0 < je; j0 += T) {
            // ---- per frequency: k_v, e_v, a_v
            const int j = j0 + tid;
            float2 a[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                           make_float2(0.f, 0.f)};
            float gam = 0.0f;
            if (j < je) {
                float sn, cs;
                sincospif((float)j / (float)L, &sn, &cs);
                const float t = sn / cs;
                gam = 2.0f * t / dt;
                float2 k[4], k2[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) k[v] = k2[v] = make_float2(0.f, 0.f);
                for (int n = 0; n < Nh; ++n) {
                    const float *w = md + kModeFloats * n;
                    const float2 r1 = crcp(make_float2(-w[0], gam - w[1]));   // 1/(s - lambda)
                    const float2 r2 = crcp(make_float2(-w[0], gam + w[1]));   // 1/(s - conj lambda)
                    const float2 q1 = cmul(r1, r1), q2 = cmul(r2, r2);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float2 vv = make_float2(w[10 + 2 * v], w[11 + 2 * v]);
                        k[v] = cadd(k[v], cadd(cmul(vv, r1), cmulc(r2, vv)));
                        k2[v] = cadd(k2[v], cadd(cmul(vv, q1), cmulc(q2, vv)));
                    }
                }
                const float2 c = make_float2(1.0f, t);
                const float2 iden = crcp(make_float2(1.0f + k[3].x, k[3].y));
                float2 e[4];
                e[0] = c;
                e[1] = cscale(cmul(c, cmul(k[2], iden)), -1.0f);
                e[2] = cscale(cmul(c, cmul(k[1], iden)), -1.0f);
                e[3] = cmul(c, cmul(cmul(k[1], k[2]), cmul(iden, iden)));
                float2 G;
                if constexpr (GG) G = gh[j];
                else G = buf[pidx(digrev_inv<LG>(j))];
                const float wj = (j == 0 ? 1.0f : 2.0f) / (float)L;
                const float2 gj = make_float2(G.x * wj, G.y * wj);
                float2 dw = make_float2(0.f, 0.f);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    a[v] = cmulc(e[v], gj);   // conj(g) e_v
                    dw = cadd(dw, cmul(e[v], k2[v]));
                }
                // dK_hat/dlog_dt = s sum_v e_v sum_i v_i r_i^2, s = i gamma
                const float2 sdw = make_float2(-gam * dw.y, gam * dw.x);
                ld_acc = fmaf(gj.x, sdw.x, fmaf(gj.y, sdw.y, ld_acc));   // Re(conj(g) sdw)
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                chA[8 * tid + 2 * v] = a[v].x;
                chA[8 * tid + 2 * v + 1] = a[v].y;
            }
            chG[tid] = gam;
            __syncthreads();
            // ---- per mode: S_v, S2_v over this chunk
            if (my_q < nq) {
                const int jn = (je - j0) < T ? (je - j0) : T;
                for (int jj = my_q; jj < jn; jj += nq) {
                    const float g = chG[jj];
                    const float2 r1 = crcp(make_float2(-lam_n.x, g - lam_n.y));
                    const float2 r2 = crcp(make_float2(-lam_n.x, g + lam_n.y));
                    const float2 q1 = cmul(r1, r1), q2 = cmul(r2, r2);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float2 av = make_float2(chA[8 * jj + 2 * v], chA[8 * jj + 2 * v + 1]);
                        S[v] = cadd(S[v], cadd(cmul(av, r2), cconj(cmul(av, r1))));
                        S2[v] = cadd(S2[v], cadd(cmul(av, q2), cconj(cmul(av, q1))));
                    }
                }
            }
            __syncthreads();
        }
        // ---- add the partial sums of each mode; the Nyquist bin; write
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            red[16 * tid + 2 * v] = S[v].x;
            red[16 * tid + 2 * v + 1] = S[v].y;
            red[16 * tid + 8 + 2 * v] = S2[v].x;
            red[16 * tid + 8 + 2 * v + 1] = S2[v].y;
        }
        if constexpr (GG) {   // the slice's per-mode sums and its dlog_dt share (no Nyquist term)
            for (int off = 16; off > 0; off >>= 1) ld_acc += __shfl_xor_sync(0xffffffffu, ld_acc, off);
            if ((tid & 31) == 0) red32[tid >> 5] = ld_acc;
            __syncthreads();
            float *pi = part + (size_t)item * (16 * Nh + 1);
            if (tid == 0) {
                float sum = 0.0f;
                for (int i = 0; i < T / 32; ++i) sum += red32[i];
                pi[16 * Nh] = sum;
            }
            for (int n = tid; n < Nh; n += T) {
                float acc[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
                for (int qq = 0; qq < nq; ++qq) {
                    const float *r = red + 16 * (qq * Nh + n);
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[i] += r[i];
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) pi[16 * n + i] = acc[i];
            }
            __syncthreads();   // shared memory is reused by the next item
            continue;
        }
        float gN;
        if constexpr (GG) gN = gh[L / 2].x / (float)L;
        else gN = buf[pidx(digrev_inv<LG>(L / 2))].x / (float)L;
        if (tid < Nh) {   // Nyquist share of dlog_dt: gN dt Re(C_n B_n), summed below
            const float *w = md + kModeFloats * tid;
            ld_acc = fmaf(gN * dt, w[10], ld_acc);
        }
        for (int off = 16; off > 0; off >>= 1) ld_acc += __shfl_xor_sync(0xffffffffu, ld_acc, off);
        if ((tid & 31) == 0) red32[tid >> 5] = ld_acc;
        __syncthreads();
        if (tid == 0) {
            float sum = 0.0f;
            for (int i = 0; i < T / 32; ++i) sum += red32[i];
            dlog_dt[h] = sum;
        }
        for (int n = tid; n < Nh; n += T) {
            float2 Sv[4], S2v[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) Sv[v] = S2v[v] = make_float2(0.f, 0.f);
            for (int qq = 0; qq < nq; ++qq) {
                const float *r = red + 16 * (qq * Nh + n);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    Sv[v] = cadd(Sv[v], make_float2(r[2 * v], r[2 * v + 1]));
                    S2v[v] = cadd(S2v[v], make_float2(r[8 + 2 * v], r[8 + 2 * v + 1]));
                }
            }
            const float *w = md + kModeFloats * n;
            const float2 c = make_float2(w[2], w[3]), b = make_float2(w[4], w[5]);
            const float2 p = make_float2(w[6], w[7]), q = make_float2(w[8], w[9]);
            float2 gC = cadd(cmulc(Sv[0], b), cmulc(Sv[1], p));      // conj(B) S00 + conj(P) S01
            float2 gB = cadd(cmulc(Sv[0], c), cmul(q, Sv[2]));       // conj(C) S00 + Q S10
            const float2 gP = cadd(cmulc(Sv[1], c), cmul(q, Sv[3]));  // conj(C) S01 + Q S11
            const float2 gQ = cadd(cmulc(b, Sv[2]), cmulc(p, Sv[3]));  // B conj(S10) + P conj(S11)
            float2 gL = make_float2(0.f, 0.f);
#pragma unroll
            for (int v = 0; v < 4; ++v) gL = cadd(gL, cmulc(S2v[v], make_float2(w[10 + 2 * v], w[11 + 2 * v])));
            gC = cadd(gC, cscale(cconj(b), gN * dt));
            gB = cadd(gB, cscale(cconj(c), gN * dt));
            dLambda[po + n] = gL;
            dP[po + n] = gP;
            dQ[po + n] = gQ;
            dB[po + n] = gB;
            dC[po + n] = gC;
        }
        __syncthreads();   // shared memory is reused by the next channel
    }
}

namespace {
struct LaunchCache {
    int resident[64];
};
template <int LG>
cudaError_t run_corr(const float *u, const float *dy, int Bt, int H, float *dK, float *dD, void *ws,
                     cudaStream_t st) {
    static LaunchCache cache;
    constexpr int T = pair_threads<LG>();
    constexpr size_t smem = pair_smem_bytes<LG>(0);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int &res = cache.resident[dev & 63];
    if (res == 0) {
        e = cudaFuncSetAttribute(k_corr_pair<LG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        int per_sm = 0, sms = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_corr_pair<LG>, T, smem);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        if (per_sm * sms <= 0) return cudaErrorInvalidConfiguration;
        res = per_sm * sms;
    }
    const size_t half = corr_workspace_bytes(H, 1 << LG) / 2;
    float2 *acc = (float2 *)ws, *zs = (float2 *)((char *)ws + half);
    k_corr_pair<LG><<<res < H ? res : H, T, smem, st>>>(u, dy, Bt, H, dK, dD, acc, zs);
    return cudaGetLastError();
}
}  // namespace

namespace {
template <int LG, bool GG = false>
cudaError_t run_kgen_backward(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B,
                              const float2 *C, const float *log_dt, const float *dK, int H, int Nh,
                              float2 *dLambda, float2 *dP, float2 *dQ, float2 *dB, float2 *dC, float *dlog_dt,
                              cudaStream_t st, const float2 *ghat = nullptr, int FS = 1, float *part = nullptr) {
    const size_t smem = kbwd_smem_bytes<LG, GG>(Nh);
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess && smem > 48 * 1024)
        e = cudaFuncSetAttribute(k_kgen_backward<LG, GG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_kgen_backward<LG, GG>, kBwdThreads, smem);
    if (e != cudaSuccess) return e;
    const int slots = (per_sm > 0 ? per_sm : 1) * sms;
    const long long items = (long long)H * (GG ? FS : 1);
    const int grid = items < slots ? (int)items : slots;
    k_kgen_backward<LG, GG><<<grid, kBwdThreads, smem, st>>>(Lambda, P, Q, B, C, log_dt, dK, ghat, H, Nh, FS, part,
                                                             dLambda, dP, dQ, dB, dC, dlog_dt);
    return cudaGetLastError();
}
}  // namespace

// frequency slices per channel for L > 16384: enough items for ~2 CTAs per
// SM of a 148-SM device, a power of two, at most 64 (fixed by H alone, so the
// workspace size does not depend on the device)
int kbwd_slices(int H) {
    int fs = 1;
    while (fs < 64 && (long long)H * fs < 296) fs *= 2;
    return fs;
}

// L > 16384: adds the FS slices of every mode in slice order, then the
// Nyquist bin, and forms the gradients (the formulas of k_kgen_backward)
__global__ void __launch_bounds__(kBwdThreads)
k_kgen_backward_assemble(const float2 *__restrict__ Lambda, const float2 *__restrict__ P,
                         const float2 *__restrict__ Q, const float2 *__restrict__ B, const float2 *__restrict__ Cc,
                         const float *__restrict__ log_dt, const float2 *__restrict__ ghat, int Nh, int L, int FS,
                         const float *__restrict__ part, float2 *__restrict__ dLambda, float2 *__restrict__ dP,
                         float2 *__restrict__ dQ, float2 *__restrict__ dB, float2 *__restrict__ dC,
                         float *__restrict__ dlog_dt) {
    __shared__ float red32[kBwdThreads / 32];
    const int h = blockIdx.x, tid = threadIdx.x;
    const float dt = expf(__ldg(log_dt + h));
    const float gN = ghat[(size_t)h * (L / 2 + 1) + L / 2].x / (float)L;
    const size_t stride = 16 * (size_t)Nh + 1;
    const float *ph = part + (size_t)h * FS * stride;
    float ld = 0.0f;
    if (tid == 0)
        for (int f = 0; f < FS; ++f) ld += ph[f * stride + 16 * Nh];
    for (int n = tid; n < Nh; n += kBwdThreads) {
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
        for (int f = 0; f < FS; ++f)
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] += ph[f * stride + 16 * n + i];
        float2 Sv[4], S2v[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            Sv[v] = make_float2(acc[2 * v], acc[2 * v + 1]);
            S2v[v] = make_float2(acc[8 + 2 * v], acc[9 + 2 * v]);
        }
        const size_t o = (size_t)h * Nh + n;
        const float2 c = Cc[o], b = B[o], p = P[o], q = Q[o];
        const float2 vv[4] = {cmul(c, b), cmul(c, p), cmulc(b, q), cmulc(p, q)};
        float2 gC = cadd(cmulc(Sv[0], b), cmulc(Sv[1], p));      // conj(B) S00 + conj(P) S01
        float2 gB = cadd(cmulc(Sv[0], c), cmul(q, Sv[2]));       // conj(C) S00 + Q S10
        const float2 gP = cadd(cmulc(Sv[1], c), cmul(q, Sv[3]));  // conj(C) S01 + Q S11
        const float2 gQ = cadd(cmulc(b, Sv[2]), cmulc(p, Sv[3]));  // B conj(S10) + P conj(S11)
        float2 gL = make_float2(0.f, 0.f);
#pragma unroll
        for (int v = 0; v < 4; ++v) gL = cadd(gL, cmulc(S2v[v], vv[v]));
        gC = cadd(gC, cscale(cconj(b), gN * dt));
        gB = cadd(gB, cscale(cconj(c), gN * dt));
        dLambda[o] = gL;
        dP[o] = gP;
        dQ[o] = gQ;
        dB[o] = gB;
        dC[o] = gC;
        ld = fmaf(gN * dt, vv[0].x, ld);   // Nyquist share: gN dt Re(C_n B_n)
    }
    for (int off = 16; off > 0; off >>= 1) ld += __shfl_xor_sync(0xffffffffu, ld, off);
    if ((tid & 31) == 0) red32[tid >> 5] = ld;
    __syncthreads();
    if (tid == 0) {
        float sum = 0.0f;
        for (int i = 0; i < kBwdThreads / 32; ++i) sum += red32[i];
        dlog_dt[h] = sum;
    }
}

// ---- DFT of dK for L >= 32768 by four steps, L = n1 n2, n1 = 256:
//   G[h, j1 + n1 j2] = sum_{k2} w_n2^{j2 k2} ( w_L^{j1 k2} sum_{k1} w_n1^{j1 k1} dK[h, n2 k1 + k2] ),
// w_n = exp(-2 pi i / n). Each kernel runs 32 sequences of one size
// n = 16 R2 (R2 = 8 or 16) per CTA in shared memory (element k of sequence c
// at k * 33 + c): with k = R2 a + b and j = p + 16 q, pass 1 takes the
// length-16 DFT over a for each b and multiplies by w_n^{b p} (in place, at
// R2 p + b), pass 2 the length-R2 DFT over b, leaving X[p + 16 q] at
// R2 p + q.
template <int R2>
__device__ void dft32_smem(float2 *s) {
    constexpr int n = 16 * R2, T = kBwdThreads;
    for (int it = threadIdx.x; it < 32 * R2; it += T) {
        const int c = it & 31, b = it >> 5;
        float2 x[16];
#pragma unroll
        for (int a = 0; a < 16; ++a) x[a] = s[(R2 * a + b) * 33 + c];
        dft<16, -1>(x);
#pragma unroll
        for (int p = 0; p < 16; ++p) s[(R2 * p + b) * 33 + c] = cmul(x[p], unit_root(b * p, n));
    }
    __syncthreads();
    for (int it = threadIdx.x; it < 32 * 16; it += T) {
        const int c = it & 31, p = it >> 5;
        float2 z[R2];
#pragma unroll
        for (int b = 0; b < R2; ++b) z[b] = s[(R2 * p + b) * 33 + c];
        dft<R2, -1>(z);
#pragma unroll
        for (int q = 0; q < R2; ++q) s[(R2 * p + q) * 33 + c] = z[q];
    }
    __syncthreads();
}
constexpr int kDftN1 = 256;

// columns: CTA (x, h) takes k2 = 32 x .. 32 x + 31; Y[h, j1, k2] = w_L^{j1 k2} X
__global__ void __launch_bounds__(kBwdThreads) k_dft_cols(const float *__restrict__ dK, int L,
                                                          float2 *__restrict__ Y) {
    extern __shared__ float2 s[];   // [kDftN1][33]
    const int h = blockIdx.y, k20 = blockIdx.x * 32, n2 = L / kDftN1;
    const float *src = dK + (size_t)h * L;
    for (int i = threadIdx.x; i < kDftN1 * 32; i += kBwdThreads) {
        const int k1 = i >> 5, c = i & 31;
        s[k1 * 33 + c] = make_float2(src[(size_t)n2 * k1 + k20 + c], 0.0f);
    }
    __syncthreads();
    dft32_smem<kDftN1 / 16>(s);
    float2 *dst = Y + (size_t)h * L;
    for (int i = threadIdx.x; i < kDftN1 * 32; i += kBwdThreads) {
        const int c = i & 31, j1 = i >> 5, p = j1 & 15, q = j1 >> 4;
        const int k2 = k20 + c;
        dst[(size_t)j1 * n2 + k2] = cmul(s[(16 * p + q) * 33 + c], unit_root((j1 * k2) & (L - 1), L));
    }
}

// rows: CTA (x, h) takes j1 = 32 x .. 32 x + 31; G[h, j1 + n1 j2] for j <= L / 2
template <int R2>
__global__ void __launch_bounds__(kBwdThreads) k_dft_rows(const float2 *__restrict__ Y, int L,
                                                          float2 *__restrict__ G) {
    constexpr int n2 = 16 * R2;
    extern __shared__ float2 s[];   // [n2][33]
    const int h = blockIdx.y, j10 = blockIdx.x * 32;
    const float2 *src = Y + (size_t)h * L;
    for (int i = threadIdx.x; i < n2 * 32; i += kBwdThreads) {
        const int k2 = i % n2, c = i / n2;
        s[k2 * 33 + c] = src[(size_t)(j10 + c) * n2 + k2];
    }
    __syncthreads();
    dft32_smem<R2>(s);
    float2 *dst = G + (size_t)h * (L / 2 + 1);
    for (int i = threadIdx.x; i < n2 * 32; i += kBwdThreads) {
        const int c = i & 31, j2 = i >> 5, p = j2 & 15, q = j2 >> 4;
        const int j = j10 + c + kDftN1 * j2;
        if (j <= L / 2) dst[j] = s[(R2 * p + q) * 33 + c];
    }
}

// Y (four-step intermediate), G_hat, and the slices' partial sums (bounded
// with Nh = S4_MAX_NH)
size_t kgen_backward_workspace_bytes(int H, int L) {
    if (L <= 16384) return 0;
    return (((size_t)H * L * sizeof(float2) + 255) & ~size_t(255)) +
           (((size_t)H * (L / 2 + 1) * sizeof(float2) + 255) & ~size_t(255)) +
           (((size_t)H * kbwd_slices(H) * (16 * (size_t)S4_MAX_NH + 1) * sizeof(float) + 255) & ~size_t(255));
}

cudaError_t launch_kgen_backward(const float2 *Lambda, const float2 *P, const float2 *Q, const float2 *B,
                                 const float2 *C, const float *log_dt, const float *dK, int H, int Nh, int L,
                                 float2 *dLambda, float2 *dP, float2 *dQ, float2 *dB, float2 *dC,
                                 float *dlog_dt, void *ws, cudaStream_t st) {
#define S4_KBWD(LG) run_kgen_backward<LG>(Lambda, P, Q, B, C, log_dt, dK, H, Nh, dLambda, dP, dQ, dB, dC, dlog_dt, st)
    if (L > 16384) {   // G_hat by the four-step DFT into the workspace, then the gradients
        float2 *Y = static_cast<float2 *>(ws);
        float2 *G = reinterpret_cast<float2 *>(static_cast<char *>(ws) +
                                               (((size_t)H * L * sizeof(float2) + 255) & ~size_t(255)));
        const int n2 = L / kDftN1;
        const size_t smc = (size_t)kDftN1 * 33 * sizeof(float2), smr = (size_t)n2 * 33 * sizeof(float2);
        cudaError_t e = cudaFuncSetAttribute(k_dft_cols, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smc);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(n2 == 128 ? k_dft_rows<8> : k_dft_rows<16>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smr);
        if (e != cudaSuccess) return e;
        k_dft_cols<<<dim3(n2 / 32, H), kBwdThreads, smc, st>>>(dK, L, Y);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (n2 == 128) k_dft_rows<8><<<dim3(kDftN1 / 32, H), kBwdThreads, smr, st>>>(Y, L, G);
        else k_dft_rows<16><<<dim3(kDftN1 / 32, H), kBwdThreads, smr, st>>>(Y, L, G);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        float *part = reinterpret_cast<float *>(reinterpret_cast<char *>(G) +
                                                (((size_t)H * (L / 2 + 1) * sizeof(float2) + 255) & ~size_t(255)));
        const int FS = kbwd_slices(H);
        e = L == 32768 ? run_kgen_backward<15, true>(Lambda, P, Q, B, C, log_dt, dK, H, Nh, dLambda, dP, dQ, dB, dC,
                                                     dlog_dt, st, G, FS, part)
                       : run_kgen_backward<16, true>(Lambda, P, Q, B, C, log_dt, dK, H, Nh, dLambda, dP, dQ, dB, dC,
                                                     dlog_dt, st, G, FS, part);
        if (e != cudaSuccess) return e;
        k_kgen_backward_assemble<<<H, kBwdThreads, 0, st>>>(Lambda, P, Q, B, C, log_dt, G, Nh, L, FS, part, dLambda,
                                                              dP, dQ, dB, dC, dlog_dt);
        return cudaGetLastError();
    }
    switch (L) {
        case 16: return S4_KBWD(4);
        case 32: return S4_KBWD(5);
        case 64: return S4_KBWD(6);
        case 128: return S4_KBWD(7);
        case 256: return S4_KBWD(8);
        case 512: return S4_KBWD(9);
        case 1024: return S4_KBWD(10);
        case 2048: return S4_KBWD(11);
        case 4096: return S4_KBWD(12);
        case 8192: return S4_KBWD(13);
        case 16384: return S4_KBWD(14);
        default: return cudaErrorInvalidValue;
    }
#undef S4_KBWD
}

namespace {
size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// dK = r (first) or dK += r (float4; n a multiple of 4)
__global__ void k_accumulate(float *__restrict__ dK, const float *__restrict__ r, size_t n4, bool first) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const float4 b = reinterpret_cast<const float4 *>(r)[i];
        if (first) {
            reinterpret_cast<float4 *>(dK)[i] = b;
        } else {
            float4 a = reinterpret_cast<float4 *>(dK)[i];
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
            reinterpret_cast<float4 *>(dK)[i] = a;
        }
    }
}
// dD[h] = dK[h, 0]
__global__ void k_lag0(const float *__restrict__ dK, int H, int L, float *__restrict__ dD) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h < H) dD[h] = dK[(size_t)h * L];
}

// L > 8192, per pair of batch rows (b, b + 1): the spectrum Z_u of the
// zero-padded complex signal u[b] + i u[b + 1] is prepared as if it were a
// kernel spectrum, and the adjoint convolution of the row pair dy[b], dy[b+1]
// (packed dy[b] + i dy[b + 1], multiplied by conj(Z_u)) has as its real part
//   sum_t dy[b,h,t] u[b,h,t-s] + sum_t dy[b+1,h,t] u[b+1,h,t-s],
// the two rows' shares of dK[h, s] (the imaginary part holds cross terms and
// goes to scratch). An odd last row uses the real spectrum of u[b] alone.
// The shares are added in batch order.
cudaError_t run_corr_long(const float *u, const float *dy, int Bt, int H, int L, float *dK, float *dD, void *ws,
                          cudaStream_t st) {
    void *spec = ws;
    float *r = reinterpret_cast<float *>(static_cast<char *>(ws) + align256(conv_workspace_bytes(H, L)));
    const size_t row = (size_t)H * L;
    cudaError_t e = cudaSuccess;
    for (int b = 0; b < Bt && e == cudaSuccess; b += 2) {
        const int nb = (b + 1 < Bt) ? 2 : 1;
        e = launch_kspec(u + b * row, nullptr, H, L, spec, st, nb == 2 ? u + (b + 1) * row : nullptr);
        if (e == cudaSuccess) e = launch_fftconv(dy + b * row, spec, nb, H, L, r, st, true);
        if (e == cudaSuccess) {
            k_accumulate<<<1184, 256, 0, st>>>(dK, r, row / 4, b == 0);
            e = cudaGetLastError();
        }
    }
    if (e == cudaSuccess && dD != nullptr) {
        k_lag0<<<(H + 255) / 256, 256, 0, st>>>(dK, H, L, dD);
        e = cudaGetLastError();
    }
    return e;
}
}  // namespace

size_t corr_workspace_bytes(int H, int L) {
    if (L > 8192) return align256(conv_workspace_bytes(H, L)) + align256((size_t)2 * H * L * sizeof(float));
    return 2 * (((size_t)H * 2 * L * sizeof(float2) + 255) & ~size_t(255));
}

cudaError_t launch_corr(const float *u, const float *dy, int Bt, int H, int L, float *dK, float *dD, void *ws,
                        cudaStream_t st) {
    switch (L) {
        case 16: return run_corr<4>(u, dy, Bt, H, dK, dD, ws, st);
        case 32: return run_corr<5>(u, dy, Bt, H, dK, dD, ws, st);
        case 64: return run_corr<6>(u, dy, Bt, H, dK, dD, ws, st);
        case 128: return run_corr<7>(u, dy, Bt, H, dK, dD, ws, st);
        case 256: return run_corr<8>(u, dy, Bt, H, dK, dD, ws, st);
        case 512: return run_corr<9>(u, dy, Bt, H, dK, dD, ws, st);
        case 1024: return run_corr<10>(u, dy, Bt, H, dK, dD, ws, st);
        case 2048: return run_corr<11>(u, dy, Bt, H, dK, dD, ws, st);
        case 4096: return run_corr<12>(u, dy, Bt, H, dK, dD, ws, st);
        case 8192: return run_corr<13>(u, dy, Bt, H, dK, dD, ws, st);
        default: return run_corr_long(u, dy, Bt, H, L, dK, dD, ws, st);
    }
}

}  // namespace s4
